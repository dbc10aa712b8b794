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
// expert) with the token positions routed to it, cut into token groups of at
// most TS tokens.  Each slot's matrix is cut into blocks of RB rows (always
// 48 KB: 384 threads x 8 rows x 16 bytes); the (slot, group, block) units are
// split into contiguous ranges of equal estimated cost (weight streaming plus
// per-token dot work), one range per CTA, one CTA per SM.
//
// Memory pipeline.  Thread 0 streams the CTA's blocks with cp.async.bulk into
// a ring of 3-4 shared-memory stages (mbarrier completion, bounded waits), so
// up to 144-192 KB per SM are in flight while the CTA computes.  Inside a CTA
// a "team" of CPR threads covers one row (thread c reads 16-byte chunk c) and
// handles R = 8 consecutive rows of a block.  Activations enter as digit
// planes (qrx_dev.cuh) prepared once per row by k_act_digits (tokens, for
// gate/up) and k_h_digits (h rows, for down); every thread loads its chunk's
// digit words straight from those records (L2-resident).  With several
// tokens per slot a pass takes TP tokens' digits into registers and reads and
// unpacks each weight chunk once for all of them (int2, whose unpacked chunk
// does not fit beside them, re-reads it per token); a token group is bounded
// only by the per-stage partial sums (64 tokens at the GLM shape), so each
// expert's weights stream once per call at decode batch sizes.  Reductions
// are fixed-order (warp butterflies, then warp partials in index order), so
// results are deterministic.  For gate/up a block holds rows of the gate
// matrix and the same rows of the up matrix (two copies into one stage), so
// the SwiGLU is applied where both sums meet.  Calls of more than four tokens
// use this engine; k_gemv2.cuh takes decode calls of up to four.
#pragma once
#include <atomic>
#include <cuda/atomic>
#include "qrx_dev.cuh"
#include "qrx_check.cuh"

namespace qrx {

constexpr int GV_BLK = 48 * 1024;             // bytes per block: NT threads x R rows x 16 B

// Threads per CTA (12 warps, 8 rows per thread).
template <int WB, int NDIG> struct GvShape {
    static constexpr int NT = 384;
    static constexpr int R = GV_BLK / (NT * 16);
};
constexpr int GV_SMEM_MAX = 227 * 1024;       // dynamic shared memory per CTA
constexpr long long GV_WAIT_CAP = 1ll << 22;  // mbarrier polls before giving up

// ---------------------------------------------------------------- records
// Digit record of one activation row of length K (per token or per h row):
//   planes [NDIG][K] bytes, chunk-permuted for the weight format (digit_slot)
//   scales [K/32] f32      (sigma_b: 2^-s for 22-bit fixed point, d_b for Q8_0)
//   corr   [K/32][NDIG] i32 (-OFF * sum of the block's digits, per plane)
__host__ __device__ constexpr int align16(int v) { return (v + 15) & ~15; }

struct RecLayout {
    int scales, corr, bytes;
};

__host__ __device__ inline RecLayout rec_layout(int ndig, int K)
{
    RecLayout L;
    L.scales = ndig * K;
    L.corr = L.scales + align16((K / 32) * 4);
    L.bytes = L.corr + align16((K / 32) * ndig * 4);
    return L;
}

// 2^s as f32 for -126 <= s <= 127, else via ldexpf.
__device__ __forceinline__ float pow2f(int s)
{
    return (s >= -126 && s <= 127) ? __int_as_float((s + 127) << 23) : ldexpf(1.f, s);
}

// Convert one 32-element block (lane = element) into the record `rec`:
// NDIG = 3: f32 value -> 3 digits of a 22-bit fixed point; NDIG = 1: Q8_0
// quantisation of the f32 value.  The caller rounds to bf16 first when the
// activations are bf16.  All 32 lanes of the warp must call.
template <int WB, int NDIG>
__device__ __forceinline__ void stage_block(unsigned char *rec, const RecLayout &L, int cpr, int b,
                                            int lane, float v)
{
    using F = Fmt<WB>;
    const float amax = warp_max(fabsf(v));
    int8_t d[3] = {0, 0, 0};
    float sig = 0.f;
    if constexpr (NDIG == 1) {
        if (amax != 0.f) {
            d[0] = (int8_t)q8_code(v, __fdiv_rn(127.f, amax));
            sig = __fdiv_rn(amax, 127.f);
        }
    } else {
        if (amax != 0.f) {
            const int sh = fixed_shift(amax);
            const float scaled = (sh >= -126 && sh <= 127) ? __fmul_rn(v, pow2f(sh)) : ldexpf(v, sh);
            split3(__float2int_rn(scaled), d[0], d[1], d[2]);
            sig = pow2f(-sh);
        }
    }
    const int elem = b * 32 + lane;
    const int cc = elem / F::EPC, l = elem % F::EPC;
    int wd, by;
    digit_slot<WB>(l, wd, by);
    const int K = cpr * F::EPC;
#pragma unroll
    for (int pl = 0; pl < NDIG; ++pl) {
        rec[(size_t)pl * K + ((size_t)cc * F::DW + wd) * 4 + by] = (unsigned char)d[pl];
        int sum = d[pl];
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) reinterpret_cast<int *>(rec + L.corr)[b * NDIG + pl] = -F::OFF * sum;
    }
    if (lane == 0) reinterpret_cast<float *>(rec + L.scales)[b] = sig;
}

// Q8_0 codes and scales already computed (qrx_quantize_act_q8): permute only.
template <int WB>
__device__ __forceinline__ void stage_block_q8(unsigned char *rec, const RecLayout &L, int cpr, int b,
                                               int lane, int8_t q, float dq)
{
    using F = Fmt<WB>;
    const int elem = b * 32 + lane;
    const int cc = elem / F::EPC, l = elem % F::EPC;
    int wd, by;
    digit_slot<WB>(l, wd, by);
    rec[((size_t)cc * F::DW + wd) * 4 + by] = (unsigned char)q;
    int sum = q;
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        reinterpret_cast<int *>(rec + L.corr)[b] = -F::OFF * sum;
        reinterpret_cast<float *>(rec + L.scales)[b] = dq;
    }
}

// Activation rows -> digit records in global memory, one warp per block of 32.
// Q8_0: from precomputed codes (xq, xd) or, when xq is null, from f32 x.
template <int WB, int NDIG>
__global__ void __launch_bounds__(256) k_act_digits(const void *__restrict__ x,
                                                    const int8_t *__restrict__ xq,
                                                    const float *__restrict__ xd, int afmt, int T,
                                                    int K, unsigned char *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int nb = K / 32;
    pdl_wait();
    pdl_trigger();
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= (int64_t)T * nb) return;
    const int t = (int)(gw / nb), b = (int)(gw % nb);
    const RecLayout L = rec_layout(NDIG, K);
    unsigned char *rec = out + (size_t)t * L.bytes;
    const int cpr = K / Fmt<WB>::EPC;
    const int64_t e = (int64_t)t * K + b * 32 + lane;
    if constexpr (NDIG == 1) {
        if (xq)          // codes and scales from qrx_quantize_act_q8
            stage_block_q8<WB>(rec, L, cpr, b, lane, xq[e], xd[(int64_t)t * nb + b]);
        else             // quantise the f32 activations here (same Q8_0 formula)
            stage_block<WB, 1>(rec, L, cpr, b, lane, reinterpret_cast<const float *>(x)[e]);
    } else {
        const float v = afmt == QRX_A_BF16
                            ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(x)[e])
                            : reinterpret_cast<const float *>(x)[e];
        stage_block<WB, NDIG>(rec, L, cpr, b, lane, v);
    }
}

// h rows (f32, row stride ld) -> digit records, one warp per block of 32; for
// bf16 activations h is rounded to bf16 first (the down projection's input).
template <int WB, int NDIG>
__global__ void __launch_bounds__(256) k_h_digits(const float *__restrict__ h, int64_t ld, int rows,
                                                  int K, int afmt, unsigned char *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int nb = K / 32;
    pdl_wait();
    pdl_trigger();
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= (int64_t)rows * nb) return;
    const int r = (int)(gw / nb), b = (int)(gw % nb);
    const RecLayout L = rec_layout(NDIG, K);
    float v = h[(int64_t)r * ld + b * 32 + lane];
    if (afmt == QRX_A_BF16) v = __bfloat162float(__float2bfloat16_rn(v));
    stage_block<WB, NDIG>(out + (size_t)r * L.bytes, L, K / Fmt<WB>::EPC, b, lane, v);
}

// ---------------------------------------------------------------- mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One bulk copy completing on `mbar` (its bytes were announced by expect_tx).
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst), "l"(src), "r"(bytes), "r"(mbar)
        : "memory");
}

// Bounded wait for phase `parity` of an mbarrier; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity)
{
    for (long long it = 0; it < GV_WAIT_CAP; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// ---------------------------------------------------------------- kernel
struct GvSmem {
    int stage_bytes, scales_off, mbar, cnt, abort, red, red_stage, pre, total;
};

// Shared memory: `stages` ring stages (weights, then the block's row scales),
// their mbarriers and arrival counters, per-stage partial sums
// [ts][tpc][wpt][R], the slot cost prefix.  Activation records stay in global
// memory (L2): every lane reads its chunk's digit words from there.
__host__ __device__ inline GvSmem gv_smem(int stages, int ts, int rb, int tpc, int wpt, int R,
                                          int maxslots)
{
    GvSmem m;
    m.scales_off = GV_BLK;
    m.stage_bytes = GV_BLK + align16(rb * 4);
    int o = stages * m.stage_bytes;
    m.mbar = o;
    o += stages * 8;
    m.cnt = o;
    o += stages * 4;
    m.abort = o;
    o = align16(o + 4);
    m.red = o;
    m.red_stage = ts * tpc * wpt * R;         // floats
    o += stages * m.red_stage * 4;
    o = (o + 7) & ~7;
    m.pre = o;
    o += (maxslots + 2) * 8;
    m.total = o;
    return m;
}

struct GemvP {
    int K, rows, row_bytes, cpr, tpc, rb, rbm, nblk, ts, wpt, stages, maxslots, nthreads;
    RecLayout rec;
    GvSmem sm;
    // matrix m of expert e: codes w[m] + e*w_stride[m] bytes, scales s[m] +
    // e*s_stride[m] floats; gate/up: m = 0 gate, 1 up (rbm rows of each per
    // block, gate rows first); down: m = 0 only (rbm = rb)
    const uint8_t *w[2];
    int64_t w_stride[2];
    const float *s[2];
    int64_t s_stride[2];
    const uint8_t *w_sh[2];
    const float *s_sh[2];
    int routed, shared;
    const int32_t *offsets, *sorted, *union_ids, *n_union;
    int E, k, T;
    int afmt;
    const unsigned char *xrec;   // digit records of the input rows (tokens, or h rows)
    int64_t sh_in_row0;          // down: record row of the shared expert's first h row
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

// A lane's view of one activation row: its chunk's digit words, block scales
// and offset corrections.
template <int WB, int NDIG>
struct LaneDig {
    static constexpr int NBC = WB == 2 ? 2 : 1;     // scale blocks touched by a chunk
    uint32_t w[NDIG][Fmt<WB>::DW];
    float sig[NBC];
    int corr[NBC][NDIG];

    __device__ __forceinline__ void load(const unsigned char *rec, const RecLayout &L, int c, int K)
    {
        constexpr int DW = Fmt<WB>::DW;
#pragma unroll
        for (int pl = 0; pl < NDIG; ++pl) {
            const uint4 *src = reinterpret_cast<const uint4 *>(rec + (size_t)pl * K + (size_t)c * DW * 4);
#pragma unroll
            for (int q = 0; q < DW / 4; ++q) {
                const uint4 v4 = src[q];
                w[pl][4 * q + 0] = v4.x;
                w[pl][4 * q + 1] = v4.y;
                w[pl][4 * q + 2] = v4.z;
                w[pl][4 * q + 3] = v4.w;
            }
        }
        const float *sc = reinterpret_cast<const float *>(rec + L.scales);
        const int *co = reinterpret_cast<const int *>(rec + L.corr);
#pragma unroll
        for (int bc = 0; bc < NBC; ++bc) {
            const int sb = WB == 8 ? (c >> 1) : (WB == 4 ? c : 2 * c + bc);
            sig[bc] = sc[sb];
#pragma unroll
            for (int pl = 0; pl < NDIG; ++pl) corr[bc][pl] = WB == 8 ? 0 : co[sb * NDIG + pl];
        }
    }

    // The same dot product on a weight chunk already unpacked (u[word][vector]):
    // the unpack is shared by every token that meets the chunk.
    __device__ __forceinline__ float dot_u(const uint32_t (&u)[4][Fmt<WB>::UPW]) const
    {
        int acc[NBC][NDIG][2];
#pragma unroll
        for (int bc = 0; bc < NBC; ++bc)
#pragma unroll
            for (int pl = 0; pl < NDIG; ++pl) {
                acc[bc][pl][0] = corr[bc][pl];
                acc[bc][pl][1] = 0;
            }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int bc = WB == 2 ? (i >> 1) : 0;
#pragma unroll
            for (int j = 0; j < Fmt<WB>::UPW; ++j)
#pragma unroll
                for (int pl = 0; pl < NDIG; ++pl)
                    acc[bc][pl][i & 1] = dp4a(u[i][j], w[pl][i * Fmt<WB>::UPW + j], acc[bc][pl][i & 1]);
        }
        float v = 0.f;
#pragma unroll
        for (int bc = 0; bc < NBC; ++bc) {
            float cv;
            if constexpr (NDIG == 3)
                cv = fmaf(__int2float_rn(acc[bc][2][0] + acc[bc][2][1]), 65536.f,
                          __int2float_rn((acc[bc][0][0] + acc[bc][0][1]) +
                                         256 * (acc[bc][1][0] + acc[bc][1][1])));
            else
                cv = __int2float_rn(acc[bc][0][0] + acc[bc][0][1]);
            v = fmaf(sig[bc], cv, v);
        }
        return v;
    }

    // The lane's share of one row's dot product: exact int32 per block, then f32.
    // Each plane keeps two partial accumulators (even and odd weight words) so
    // the dp4a chains are half as deep.
    __device__ __forceinline__ float dot(const uint4 &wv) const
    {
        int acc[NBC][NDIG][2];
#pragma unroll
        for (int bc = 0; bc < NBC; ++bc)
#pragma unroll
            for (int pl = 0; pl < NDIG; ++pl) {
                acc[bc][pl][0] = corr[bc][pl];
                acc[bc][pl][1] = 0;
            }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t u[Fmt<WB>::UPW];
            unpack_word<WB>(word_of(wv, i), u);
            const int bc = WB == 2 ? (i >> 1) : 0;
#pragma unroll
            for (int j = 0; j < Fmt<WB>::UPW; ++j)
#pragma unroll
                for (int pl = 0; pl < NDIG; ++pl)
                    acc[bc][pl][i & 1] = dp4a(u[j], w[pl][i * Fmt<WB>::UPW + j], acc[bc][pl][i & 1]);
        }
        float v = 0.f;
#pragma unroll
        for (int bc = 0; bc < NBC; ++bc) {
            float cv;
            if constexpr (NDIG == 3)
                cv = fmaf(__int2float_rn(acc[bc][2][0] + acc[bc][2][1]), 65536.f,
                          __int2float_rn((acc[bc][0][0] + acc[bc][0][1]) +
                                         256 * (acc[bc][1][0] + acc[bc][1][1])));
            else
                cv = __int2float_rn(acc[bc][0][0] + acc[bc][0][1]);
            v = fmaf(sig[bc], cv, v);
        }
        return v;
    }
};

// Iterator over the CTA's (slot, token group, block) units, in order.
struct Units {
    const int64_t *pre;
    int nslots, nu, nblk, ts;
    int64_t c0, c1, bwu;
    int s, j, ntok, nt;
    int64_t b, bend;
    bool valid;
    const uint8_t *W[2];     // the slot's weights and row scales, looked up once per slot
    const float *S[2];
};

__device__ __forceinline__ int slot_ntok(const GemvP &p, int s, int nu)
{
    if (s < nu) {
        const int e = p.union_ids[s];
        return (e >= 0 && e < p.E) ? p.offsets[e + 1] - p.offsets[e] : 0;
    }
    return p.T;
}

__device__ __forceinline__ const uint8_t *slot_weights(const GemvP &p, int s, int nu, int m);
__device__ __forceinline__ const float *slot_scales(const GemvP &p, int s, int nu, int m);

// Enter slot s: token count and the slot's weight / scale base pointers.
__device__ __forceinline__ void units_enter_slot(Units &u, const GemvP &p, int s)
{
    u.s = s;
    u.j = -1;
    if (s < u.nslots) {
        u.ntok = slot_ntok(p, s, u.nu);
        u.W[0] = slot_weights(p, s, u.nu, 0);
        u.S[0] = slot_scales(p, s, u.nu, 0);
        u.W[1] = slot_weights(p, s, u.nu, 1);
        u.S[1] = slot_scales(p, s, u.nu, 1);
    }
}

__device__ void units_advance(Units &u, const GemvP &p)
{
    if (u.valid && ++u.b < u.bend) return;
    u.valid = false;
    for (;;) {
        if (u.s >= u.nslots || u.pre[u.s] >= u.c1) return;
        ++u.j;
        if ((int64_t)u.j * u.ts >= u.ntok) {
            units_enter_slot(u, p, u.s + 1);
            continue;
        }
        const int nt = min(u.ts, u.ntok - u.j * u.ts);
        const int64_t gstart = u.pre[u.s] + (int64_t)u.nblk * u.j * (u.bwu + u.ts);
        const int64_t cb = u.bwu + nt;
        int64_t bf = u.c0 > gstart ? (u.c0 - gstart + cb - 1) / cb : 0;
        int64_t be = u.c1 > gstart ? (u.c1 - gstart + cb - 1) / cb : 0;
        if (be > u.nblk) be = u.nblk;
        if (bf < be) {
            u.b = bf;
            u.bend = be;
            u.nt = nt;
            u.valid = true;
            return;
        }
    }
}

__device__ __forceinline__ const float *slot_scales(const GemvP &p, int s, int nu, int m)
{
    if (s < nu) {
        int e = p.union_ids[s];
        e = (e >= 0 && e < p.E) ? e : 0;
        return (m ? p.s[1] : p.s[0]) + (int64_t)e * (m ? p.s_stride[1] : p.s_stride[0]);
    }
    return m ? p.s_sh[1] : p.s_sh[0];
}

__device__ __forceinline__ const uint8_t *slot_weights(const GemvP &p, int s, int nu, int m)
{
    if (s < nu) {
        int e = p.union_ids[s];
        e = (e >= 0 && e < p.E) ? e : 0;     // a bad index was flagged when the slot was costed
        return (m ? p.w[1] : p.w[0]) + (int64_t)e * (m ? p.w_stride[1] : p.w_stride[0]);
    }
    return m ? p.w_sh[1] : p.w_sh[0];
}

template <int WB, int NDIG, int TP, bool GATEUP>
__global__ void __launch_bounds__(GvShape<WB, NDIG>::NT, 1) k_ffn_gemv(const GemvP p)
{
    using LD = LaneDig<WB, NDIG>;
    constexpr int NT = GvShape<WB, NDIG>::NT;
    constexpr int R = GvShape<WB, NDIG>::R, V = R * TP, LV = Log2<V>::value;
    constexpr int NWARPS = NT / 32;
    constexpr int64_t BWU = NDIG == 1 ? 8 : 3;       // cost of streaming a block, in tokens
    extern __shared__ __align__(128) unsigned char smem[];
    const GvSmem M = p.sm;
    unsigned char *ring = smem;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + M.mbar);
    int *cnt = reinterpret_cast<int *>(smem + M.cnt);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + M.abort);
    float *red = reinterpret_cast<float *>(smem + M.red);
    int64_t *pre = reinterpret_cast<int64_t *>(smem + M.pre);

    const int tid = threadIdx.x, lane = tid & 31;
    const int K = p.K, cpr = p.cpr;
    const int c = tid % cpr, team = tid / cpr, wit = c >> 5;
    const RecLayout RL = p.rec;

    // gate/up reads the permutation and the activation records of the kernels
    // before it; down only needs h after its weight stream has started.
    if constexpr (GATEUP) {
        pdl_wait();
        pdl_trigger();
    }
    // ---- cost prefix over slots: a unit costs BWU + its token count; slot s
    // has ceil(ntok/TS) groups (all full but the last): nblk * (BWU*groups + ntok).
    const int nu = p.routed ? *p.n_union : 0;
    const int nslots = nu + (p.shared ? 1 : 0);
    QRX_CHECK_ONLY(const int64_t n_pos = p.routed ? (int64_t)p.T * p.k : 0;)   // routed positions
    QRX_CHECK_ONLY(const int64_t n_in = GATEUP ? (int64_t)p.T : max(n_pos, p.shared ? p.sh_in_row0 + p.T : (int64_t)0);)
    QRX_CHECK_ONLY(const int64_t n_out = max(n_pos, p.shared ? p.sh_out_row0 + p.T : (int64_t)0);)
    if (tid < 32) {
        int64_t run = 0;
        for (int s0 = 0; s0 < nslots; s0 += 32) {
            const int s = s0 + lane;
            int64_t cost = 0;
            if (s < nslots) {
                if (s < nu) {
                    const int e = p.union_ids[s];
                    if (e < 0 || e >= p.E) raise_status(DERR_BADIDX);
                }
                const int ntok = slot_ntok(p, s, nu);
                cost = (int64_t)p.nblk * (BWU * ((ntok + p.ts - 1) / p.ts) + ntok);
            }
            int64_t inc = cost;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t nb = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += nb;
            }
            if (s < nslots) pre[s] = run + inc - cost;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pre[nslots] = run;
    }
    if (tid == 0) {
        for (int st = 0; st < p.stages; ++st) {
            mbar_init(smem_u32(&mbar[st]), 1);
            cnt[st] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t Ctot = pre[nslots];
    Units cu;
    cu.pre = pre;
    cu.nslots = nslots;
    cu.nu = nu;
    cu.nblk = p.nblk;
    cu.ts = p.ts;
    cu.bwu = BWU;
    cu.c0 = Ctot * blockIdx.x / gridDim.x;
    cu.c1 = Ctot * (blockIdx.x + 1) / gridDim.x;
    {   // last slot whose prefix is <= c0
        int lo = 0, hi = nslots;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= cu.c0) lo = mid; else hi = mid;
        }
        cu.s = lo;
    }
    cu.ntok = 0;
    cu.W[0] = cu.W[1] = nullptr;
    cu.S[0] = cu.S[1] = nullptr;
    units_enter_slot(cu, p, cu.s);
    cu.nt = 0;
    cu.b = cu.bend = 0;
    cu.valid = false;
    units_advance(cu, p);

    // Every thread keeps a producer iterator `stages` units ahead of its own
    // consumer iterator; the last warp to finish unit n refills its stage with
    // unit n + stages.  Thread 0 issues the first `stages` units.
    // A block holds rbm rows of each matrix: gate rows, then the same up rows.
    auto issue = [&](const Units &u, int stage) {
        constexpr int NMAT = GATEUP ? 2 : 1;
        const int64_t row0 = u.b * (int64_t)p.rbm;
        const int64_t nrows = min((int64_t)p.rbm, (int64_t)p.rows - row0);
        unsigned char *dst = ring + (size_t)stage * M.stage_bytes;
        const uint32_t mb = smem_u32(&mbar[stage]);
        const uint32_t wbytes = (uint32_t)(nrows * p.row_bytes), sbytes = (uint32_t)(nrows * 4);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb),
                     "r"(NMAT * (wbytes + sbytes))
                     : "memory");
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            bulk_copy(smem_u32(dst + (size_t)m * p.rbm * p.row_bytes), u.W[m] + row0 * p.row_bytes, wbytes, mb);
            bulk_copy(smem_u32(dst + M.scales_off + m * p.rbm * 4), u.S[m] + row0, sbytes, mb);
        }
    };
    Units pu = cu;
    for (int st = 0; st < p.stages && pu.valid; ++st) {
        if (tid == 0) issue(pu, st);
        units_advance(pu, p);
    }
    if constexpr (!GATEUP) {     // the weights are on their way; now wait for h
        pdl_wait();
        pdl_trigger();
    }

    int n = 0, cur_s = -1, cur_j = -1;
    int p0 = 0, tout1 = 0, tg = 0;
    bool is_routed = false;
    LD dreg;
    // token i of the current slot: its activation record row and its output row
    auto row_in_of = [&](int i) -> int {
        QRX_CHECK_OR(!is_routed || (int64_t)p0 + i < n_pos, return 0);
        QRX_CHECK_OR(!is_routed || !GATEUP || (p.sorted[p0 + i] >= 0 && p.sorted[p0 + i] / p.k < n_in), return 0);
        if (is_routed) return GATEUP ? p.sorted[p0 + i] / p.k : p0 + i;
        return GATEUP ? i : (int)p.sh_in_row0 + i;
    };
    auto row_out_of = [&](int i) -> int { return is_routed ? p0 + i : (int)p.sh_out_row0 + i; };
    while (cu.valid) {
        const int nt = cu.nt;
        if (cu.s != cur_s || cu.j != cur_j) {
            if (cu.s != cur_s) {
                is_routed = cu.s < nu;
                if (is_routed) {
                    int e = p.union_ids[cu.s];
                    e = (e >= 0 && e < p.E) ? e : 0;
                    p0 = p.offsets[e];
                } else {
                    p0 = 0;
                }
            }
            tg = cu.j * p.ts;
            if constexpr (TP == 1) {               // one token: its record straight from global
                dreg.load(p.xrec + (size_t)row_in_of(tg) * RL.bytes, RL, c, K);
                tout1 = row_out_of(tg);
            }
            cur_s = cu.s;
            cur_j = cu.j;
        }
        const int stage = n % p.stages;
        if (!mbar_wait(smem_u32(&mbar[stage]), (uint32_t)((n / p.stages) & 1))) {
            *abort_flag = 1;
            raise_status(DERR_TIMEOUT);
            break;
        }
        const unsigned char *sbase = ring + (size_t)stage * M.stage_bytes;
        const unsigned char *blk = sbase + (size_t)team * R * p.row_bytes + (size_t)c * 16;
        float *rst = red + (size_t)stage * M.red_stage;
        for (int t0 = 0; t0 < nt; t0 += TP) {
            float part[V];
            if constexpr (TP == 1) {
                uint4 wv[R];
#pragma unroll
                for (int r = 0; r < R; ++r)
                    wv[r] = *reinterpret_cast<const uint4 *>(blk + (size_t)r * p.row_bytes);
#pragma unroll
                for (int r = 0; r < R; ++r) part[r] = dreg.dot(wv[r]);
            } else if constexpr (WB == 2) {
                // int2: the unpacked chunk (16 words) does not fit beside TP tokens'
                // digits, so each token re-reads and unpacks the chunk
#pragma unroll
                for (int tt = 0; tt < TP; ++tt) {
                    if (t0 + tt < nt) {
                        LD d;
                        d.load(p.xrec + (size_t)row_in_of(tg + t0 + tt) * RL.bytes, RL, c, K);
#pragma unroll
                        for (int r = 0; r < R; ++r)
                            part[r * TP + tt] =
                                d.dot(*reinterpret_cast<const uint4 *>(blk + (size_t)r * p.row_bytes));
                    } else {
#pragma unroll
                        for (int r = 0; r < R; ++r) part[r * TP + tt] = 0.f;
                    }
                }
            } else {
                // the pass's tokens (a missing one repeats the last, its sums discarded)
                LD d[TP];
#pragma unroll
                for (int tt = 0; tt < TP; ++tt)
                    d[tt].load(p.xrec + (size_t)row_in_of(tg + min(t0 + tt, nt - 1)) * RL.bytes, RL, c, K);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint4 wv = *reinterpret_cast<const uint4 *>(blk + (size_t)r * p.row_bytes);
                    uint32_t u[4][Fmt<WB>::UPW];
#pragma unroll
                    for (int i = 0; i < 4; ++i) unpack_word<WB>(word_of(wv, i), u[i]);
#pragma unroll
                    for (int tt = 0; tt < TP; ++tt) part[r * TP + tt] = d[tt].dot_u(u);
                }
#pragma unroll
                for (int tt = 0; tt < TP; ++tt)
                    if (t0 + tt >= nt)
#pragma unroll
                        for (int r = 0; r < R; ++r) part[r * TP + tt] = 0.f;
            }
            // warp partials of this pass -> rst[token][team][wit][row]
            if (cpr >= 32) {
                const float tot = warp_tr_reduce<V>(part, lane);
                const int vi = lane >> (5 - LV);
                const int r = vi / TP, tt = vi % TP;
                if ((lane & ((1 << (5 - LV)) - 1)) == 0 && t0 + tt < nt)
                    rst[(((t0 + tt) * p.tpc + team) * p.wpt + wit) * R + r] = tot;
            } else {
#pragma unroll
                for (int vi = 0; vi < V; ++vi) {
                    float xv = part[vi];
                    for (int o = cpr >> 1; o; o >>= 1) xv += __shfl_xor_sync(0xffffffffu, xv, o);
                    const int r = vi / TP, tt = vi % TP;
                    if (c == 0 && t0 + tt < nt) rst[((t0 + tt) * p.tpc + team) * R + r] = xv;
                }
            }
        }
        // ---- arrive; the last warp of this unit finalizes it and refills the stage.
        // __syncwarp orders the warp's partial sums before lane 0's release; the
        // last warp's acquire, then __syncwarp, orders its reads after everyone's.
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            cuda::atomic_ref<int, cuda::thread_scope_block> arrivals(cnt[stage]);
            last = arrivals.fetch_add(1, cuda::memory_order_acq_rel) == NWARPS - 1;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            __syncwarp();
            const float *scl = reinterpret_cast<const float *>(sbase + M.scales_off);
            const int rblk = (int)cu.b;
            if constexpr (GATEUP) {
                // gate row q of the block is local row q, its up row is local row rbm + q
                const int rbm = p.rbm;
                for (int f = lane; f < nt * rbm; f += 32) {
                    const int t = f / rbm, q = f % rbm;
                    const int row = rblk * rbm + q;
                    if (row >= p.rows) continue;
                    const int gl = q, ul = q + rbm;
                    const float *gsrc = rst + ((t * p.tpc + gl / R) * p.wpt) * R + gl % R;
                    const float *usrc = rst + ((t * p.tpc + ul / R) * p.wpt) * R + ul % R;
                    float G = 0.f, U = 0.f;
                    for (int w2 = 0; w2 < p.wpt; ++w2) {
                        G += gsrc[w2 * R];
                        U += usrc[w2 * R];
                    }
                    const int orow = TP == 1 ? tout1 : row_out_of(tg + t);
                    QRX_CHECK_OR(orow >= 0 && orow < n_out, continue);
                    p.out[(int64_t)orow * p.out_ld + row] = silu_mul(scl[gl] * G, scl[ul] * U);
                }
            } else {
                const int per = p.tpc * R;
                for (int f = lane; f < nt * per; f += 32) {
                    const int t = f / per, lrow = f % per;
                    const int tf = lrow / R, r = lrow % R;
                    const int row = rblk * p.rb + lrow;
                    if (row >= p.rows) continue;
                    const float *src = rst + ((t * p.tpc + tf) * p.wpt) * R;
                    float Y = 0.f;
                    for (int w2 = 0; w2 < p.wpt; ++w2) Y += src[w2 * R + r];
                    const int orow = TP == 1 ? tout1 : row_out_of(tg + t);
                    QRX_CHECK_OR(orow >= 0 && orow < n_out, continue);
                    p.out[(int64_t)orow * p.out_ld + row] = scl[lrow] * Y;
                }
            }
            __syncwarp();
            if (lane == 0) {
                cnt[stage] = 0;
                if (pu.valid) issue(pu, stage);
            }
        }
        units_advance(pu, p);
        ++n;
        units_advance(cu, p);
    }
    if (*abort_flag && tid == 0) {
        // a wait gave up: wait (bounded) for this CTA's copies still in flight
        for (int m = n; m < n + p.stages; ++m)
            mbar_wait(smem_u32(&mbar[m % p.stages]), (uint32_t)((m / p.stages) & 1));
    }
}

// ---------------------------------------------------------------- host side
struct GemvPlan {
    GemvP p;
    size_t smem;
    int tp;
};

// Geometry for a matrix of `rows` x `K` codes at `wbits`, slots of at most
// `maxtok` tokens, NDIG digit planes.  Picks the deepest weight ring and the
// largest token group that fit in shared memory.
static inline bool gemv_plan(GemvPlan &pl, int wbits, int ndig, int K, int rows, int nm, int maxtok,
                             int maxslots)
{
    GemvP &p = pl.p;
    const int NT = GvShape<4, 3>::NT;
    const int R = GV_BLK / (NT * 16);
    p.nthreads = NT;
    p.K = K;
    p.rows = rows;
    p.row_bytes = K * wbits / 8;
    p.cpr = p.row_bytes / 16;
    if (p.cpr <= 0 || p.row_bytes % 16 != 0 || NT % p.cpr != 0) return false;
    if (p.cpr < 32 && (32 % p.cpr) != 0) return false;
    if (p.cpr > 32 && (p.cpr % 32) != 0) return false;
    p.tpc = NT / p.cpr;
    p.rb = p.tpc * R;
    p.rbm = nm == 2 ? p.rb / 2 : p.rb;        // rows of each matrix per block
    p.nblk = (rows + p.rbm - 1) / p.rbm;
    p.wpt = p.cpr >= 32 ? p.cpr / 32 : 1;
    if (p.rb * 4 % 16 != 0) return false;
    pl.tp = maxtok <= 1 ? 1 : (ndig == 1 ? 4 : 2);
    p.rec = rec_layout(ndig, K);
    p.maxslots = maxslots;
    const int tries[3] = {4, 3, 2};
    for (int i = (maxtok <= 1 ? 0 : 1); i < 3; ++i) {
        const int stages = tries[i];
        // activation records are read from global memory (L2), not staged: a
        // token group is bounded only by the per-stage partial sums
        auto total = [&](int ts) {
            return gv_smem(stages, ts, p.rb, p.tpc, p.wpt, R, maxslots).total;
        };
        if (total(1) > GV_SMEM_MAX) continue;
        int ts = maxtok;
        const int per = total(2) - total(1);
        if (total(1) + (int64_t)(ts - 1) * per > GV_SMEM_MAX) ts = 1 + (GV_SMEM_MAX - total(1)) / per;
        while (ts > 1 && total(ts) > GV_SMEM_MAX) --ts;
        p.stages = stages;
        p.ts = ts;
        p.sm = gv_smem(stages, ts, p.rb, p.tpc, p.wpt, R, maxslots);
        pl.smem = (size_t)p.sm.total;
        return true;
    }
    return false;
}

template <int WB, int NDIG, int TP, bool GU>
static cudaError_t gemv_go(const GemvPlan &pl, int grid, cudaStream_t st)
{
    auto kern = k_ffn_gemv<WB, NDIG, TP, GU>;
    static std::atomic<unsigned long long> configured{0};   // bit per device: max dynamic smem set
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !(configured.load(std::memory_order_acquire) >> dev & 1ull)) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM_MAX);
        if (err != cudaSuccess) return err;
        if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
    }
    return launch_k(kern, dim3(grid), dim3(GvShape<WB, NDIG>::NT), pl.smem, st, pl.p);
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
}

// Bytes of the digit records of `rows` activation rows of length K.
static inline size_t act_records_bytes(int afmt, int K, int rows)
{
    return (size_t)rows * rec_layout(afmt == QRX_A_Q8_0 ? 1 : 3, K).bytes;
}

cudaError_t launch_act_digits(const FfnArgs &a, cudaStream_t st)
{
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    const int64_t warps = (int64_t)a.T * (a.H / 32);
    const unsigned grid = (unsigned)((warps + 7) / 8);
#define QRX_AD(WB, ND) \
    if (a.wbits == WB && ndig == ND) \
        return launch_k(k_act_digits<WB, ND>, dim3(grid), dim3(256), 0, st, a.x, a.xq, a.xd, a.afmt, \
                        a.T, a.H, a.xrec);
    QRX_AD(4, 3) QRX_AD(4, 1) QRX_AD(8, 3) QRX_AD(8, 1) QRX_AD(2, 3) QRX_AD(2, 1)
#undef QRX_AD
    return cudaErrorInvalidValue;
}

cudaError_t launch_ffn_gateup(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (ffn_use_tc(a)) return launch_ffn_tc_gateup(a, num_sms, st);
    if (a.T >= 2 && gm_use(a)) return launch_gm_gateup(a, num_sms, st);
    if (g2_use(a)) return launch_g2_gateup(a, num_sms, st);
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    GemvPlan pl;
    if (!gemv_plan(pl, a.wbits, ndig, a.H, a.I, 2, a.T, a.E + 1)) return cudaErrorInvalidValue;
    if (a.prep_records) {
        const cudaError_t err = launch_act_digits(a, st);
        if (err != cudaSuccess) return err;
    }
    GemvP &p = pl.p;
    gemv_common(p, a);
    p.w[0] = a.gate.q;
    p.w[1] = a.up.q;
    p.w_stride[0] = a.gate.sq;
    p.w_stride[1] = a.up.sq;
    p.s[0] = a.gate.s;
    p.s[1] = a.up.s;
    p.s_stride[0] = a.gate.ss;
    p.s_stride[1] = a.up.ss;
    p.w_sh[0] = a.gate_sh.q;
    p.w_sh[1] = a.up_sh.q;
    p.s_sh[0] = a.gate_sh.s;
    p.s_sh[1] = a.up_sh.s;
    p.xrec = a.xrec;
    p.sh_in_row0 = 0;
    p.out = a.h;
    p.out_ld = a.h_ld;
    p.sh_out_row0 = a.sh_h_row0;
    return gemv_dispatch<true>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_ffn_down(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (ffn_use_tc(a)) return launch_ffn_tc_down(a, num_sms, st);
    if (a.T >= 2 && gm_use(a)) return launch_gm_down(a, num_sms, st);
    if (g2_use(a)) return launch_g2_down(a, num_sms, st);
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    GemvPlan pl;
    if (!gemv_plan(pl, a.wbits, ndig, a.I, a.H, 1, a.T, a.E + 1)) return cudaErrorInvalidValue;
    GemvP &p = pl.p;
    gemv_common(p, a);
    p.w[0] = p.w[1] = a.down.q;
    p.w_stride[0] = p.w_stride[1] = a.down.sq;
    p.s[0] = p.s[1] = a.down.s;
    p.s_stride[0] = p.s_stride[1] = a.down.ss;
    p.w_sh[0] = p.w_sh[1] = a.down_sh.q;
    p.s_sh[0] = p.s_sh[1] = a.down_sh.s;
    // h rows -> digit records (all rows the down projection reads)
    const int hrows = max(a.routed ? a.T * a.k : 0, a.shared ? (int)a.sh_h_row0 + a.T : 0);
    {
        const int64_t warps = (int64_t)hrows * (a.I / 32);
        const unsigned grid = (unsigned)((warps + 7) / 8);
        cudaError_t err = cudaErrorInvalidValue;
#define QRX_HD(WB, ND) \
        if (a.wbits == WB && ndig == ND) \
            err = launch_k(k_h_digits<WB, ND>, dim3(grid), dim3(256), 0, st, (const float *)a.h, a.h_ld, \
                           hrows, a.I, a.afmt, a.hrec);
        QRX_HD(4, 3) QRX_HD(4, 1) QRX_HD(8, 3) QRX_HD(8, 1) QRX_HD(2, 3) QRX_HD(2, 1)
#undef QRX_HD
        if (err != cudaSuccess) return err;
    }
    p.xrec = a.hrec;
    p.sh_in_row0 = a.sh_h_row0;
    p.out = a.y;
    p.out_ld = a.y_ld;
    p.sh_out_row0 = a.sh_y_row0;
    return gemv_dispatch<false>(pl, a.wbits, ndig, num_sms, st);
}

}  // namespace qrx
