// k_gemv2.cuh -- decode-shaped expert FFN: calls of at most four tokens, so
// at most four tokens per expert, streamed from HBM at close to its bandwidth.
//
// README "JustVugg/colibri", section "已实现的功能": the batch-union MoE (each
// unique expert of a batch read once and applied to all positions routed to
// it), int8 / packed int4 / packed int2 weights with per-row scales
// dequantised on use, Q8_0-style int8-activation integer dots; blog "GLM-5.2
// on slow computers", section "核心技巧": a token costs the expert bytes it
// reads.  The expert is a SwiGLU FFN: h = silu(s_g Q_g x) * (s_u Q_u x), then
// y = s_d Q_d h.
//
// Work.  A unit is (slot, block of RB rows): a slot is one expert of the
// union (or the shared expert) with its tokens; for gate/up a unit holds RB
// gate rows and the same RB up rows, so the SwiGLU is applied where both sums
// meet.  Units are cut into contiguous ranges of equal estimated cost, one
// range per CTA, one CTA of 16 warps per SM.
//
// A warp owns R rows of each matrix of a unit for the whole of K: lane l
// reads 16-byte chunks l, l + 32, ... of its rows straight from HBM (128-bit
// loads that skip L1, the next chunk's loads issued before the current chunk
// is computed), unpacks the codes in registers and dots them with the
// activation digits (dp4a); its integer sums run over all of K, and the unit
// ends with one transposed warp butterfly and the epilogue (row scales,
// SwiGLU).  Rows of fewer than 32 chunks are covered by LPR = chunks lanes
// each, several rows per warp.  No weight staging, no barrier and no partial
// sum crosses warps in the streaming loop.
//
// Activations.  Every input row (a token of x for gate/up, a row of h for
// down) is turned into a "record" in shared memory by the CTA: NDIG digit
// planes of signed bytes in the order the unpacked weight words use, so each
// dot of 4 codes by 4 digits is one dp4a with an exact int32 sum.
//   NDIG = 3 (f32, bf16 inputs): one power-of-two scale per row, sigma =
//     2^-s with max|x| * 2^s in [2^21, 2^22), and x*2^s rounded to an integer
//     split into three balanced bytes (x ~= sigma (d0 + 2^8 d1 + 2^16 d2),
//     error <= 2^-22 of the row's largest magnitude).  A lane's sums per plane
//     over its chunks are exact int32; the planes are combined once per unit.
//   NDIG = 1 (Q8_0): the record holds the Q8_0 codes and per-block scales d_b
//     (README: Q8_0-style int8 activations, blocks of 32 with an f32 absmax
//     scale); every 32-block's int32 accumulator is exact and is scaled by d_b
//     in f32.
// Packed int4 / int2 fields are flipped to offset binary (code + 8, code + 2)
// by the unpack; the offset is removed through the digit sums kept in the
// record (per block for Q8_0, per chunk and plane for NDIG = 3).
#pragma once
#include "qrx_dev.cuh"
#include "qrx_check.cuh"

namespace qrx {

constexpr int G2_NW = 16;                         // warps per CTA
constexpr int G2_THREADS = 32 * G2_NW;
constexpr int G2_TMAX = 4;                        // tokens per call
constexpr int G2_SMEM_MAX = 227 * 1024;
constexpr long long G2_WAIT_CAP = 1ll << 21;      // polls before a wait gives up
constexpr uint32_t G2_SUSPEND_NS = 1000;          // a waiting thread sleeps up to this long per poll

// ---------------------------------------------------------------- records
// Record of one input row of K codes, in shared memory:
//   digits: piece (pl, q, c) = 16 bytes at ((pl * NQ + q) * cpr + c) * 16: the
//           q-th group of four digit words of chunk c in plane pl (NQ = DW/4)
//   NDIG = 3: then float sigma (16 bytes), then int csum[cpr][4]: the sums of
//             chunk c's digits in planes 0, 1, 2 (and a zero)
//   NDIG = 1: then float d[K/32] (block scales), int corr[K/32]
//             (corr_b = -OFF * sum of the block's codes)
struct G2Rec {
    int hdr, csum, bytes;
};
__host__ __device__ inline G2Rec g2_rec(int ndig, int K, int cpr)
{
    G2Rec r;
    r.hdr = ndig * K;
    r.csum = r.hdr + 16;
    r.bytes = ndig == 3 ? r.csum + cpr * 16 : r.hdr + 2 * (((K / 32) * 4 + 15) & ~15);
    return r;
}

// ---------------------------------------------------------------- parameters
struct G2Mat {
    const uint8_t *q;      // codes of expert 0, rows of row_bytes
    const float *s;        // row scales of expert 0
    int64_t sq, ss;        // expert strides: bytes, floats
};

struct G2P {
    int K, rows, row_bytes, cpr;     // codes per input row, rows per matrix, bytes per row, chunks per row
    int lpr, gpw, nj;                // lanes per row, row groups per warp, chunks per lane per row
    int rw, rb, nrb;                 // rows per warp, rows per unit (per matrix), units per slot
    int rec_bytes, rec_off, nrec;    // record size, smem offset, records held
    int bar_off, pre_off, red_off, smem;
    G2Mat m[2], msh[2];              // gate/up: m[0] gate, m[1] up; down: m[0] down
    int routed, shared;
    const int32_t *offsets, *sorted, *union_ids, *n_union;
    int E, k, T;
    int afmt;
    const void *x;                   // gate/up: x [T][K] (f32 or bf16); down: h f32 rows
    const int8_t *xq;                // gate/up Q8_0: precomputed codes [T][K] (null: quantise x)
    const float *xd;                 //              and block scales [T][K/32]
    int64_t in_ld;                   // row stride of x / h (elements)
    int64_t sh_in_row0;              // down: h row of the shared expert's first token
    float *out;
    int64_t out_ld, sh_out_row0;
    int32_t *probe;                  // Q8_0: int32 block sums [pos][nmat][rows][K/32] (may be null)
};

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t g2_smem(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool g2_try(uint32_t mbar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    return done != 0;
}

// dp4a of unsigned weight bytes by signed digit bytes: int4 high halves are
// kept in place (16 x the code), which needs the unsigned form.
__device__ __forceinline__ int g2_dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Bounded wait; false if it gave up or another role raised the abort flag.
// Each poll may suspend the thread (up to G2_SUSPEND_NS) until the phase
// completes, so a waiting warp takes no issue slots from the working ones.
__device__ __forceinline__ bool g2_wait(uint32_t mbar, uint32_t parity, volatile int *abort_flag)
{
    for (long long it = 0; it < G2_WAIT_CAP; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(mbar), "r"(parity), "r"(G2_SUSPEND_NS)
            : "memory");
        if (done) return true;
        if (*abort_flag) return false;
    }
    *abort_flag = 1;
    raise_status(DERR_TIMEOUT);
    return false;
}

// Barrier of the compute warps: lane 0 of each warp arrives on an mbarrier of
// G2_NW arrivals and every lane waits, bounded, for the phase.  `ph` is the
// caller's phase bit.  False if the wait gave up.
__device__ __forceinline__ bool g2_cbar(uint64_t *bar, uint32_t &ph, volatile int *abort_flag)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(g2_smem(bar));
    const bool ok = g2_wait(g2_smem(bar), ph, abort_flag);
    ph ^= 1u;
    return ok;
}

// a[i] for a run-time i < N without indexing a register array
template <int N, typename T>
__device__ __forceinline__ T g2_pick(const T (&a)[N], int i)
{
    T r = a[0];
#pragma unroll
    for (int q = 1; q < N; ++q)
        if (i == q) r = a[q];
    return r;
}

// Transposed butterfly over the LPR lanes of a row group.  In: V values per
// lane.  Out: with V <= LPR, lane c of the group holds the group total of
// value c / (LPR / V) in v[0]; with V > LPR, it holds those of values
// c * (V / LPR) + q in v[q], q < V / LPR.
template <int N>
__device__ __forceinline__ void g2_tr_step(float *v, int lane, int off)
{
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        const float send = up ? v[i] : v[i + N / 2];
        const float keep = up ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
}

template <int N, int OFF>
__device__ __forceinline__ void g2_tr_rec(float *v, int lane)
{
    if constexpr (OFF >= 1) {
        if constexpr (N > 1) {
            g2_tr_step<N>(v, lane, OFF);
            g2_tr_rec<N / 2, OFF / 2>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
            g2_tr_rec<1, OFF / 2>(v, lane);
        }
    }
}

template <int V, int LPR>
__device__ __forceinline__ void g2_tr_reduce(float (&v)[V], int lane)
{
    g2_tr_rec<V, LPR / 2>(v, lane);
}

// ---------------------------------------------------------------- record builder
// Element values of one input row as the dot sees them, loaded 16 bytes at a
// time: f32 rows (x, or h -- rounded to bf16 first for bf16 activations) or
// bf16 rows (x).
struct G2Row {
    const void *base;     // the row
    bool bf16_in;         // the row is bf16 (gate/up input with bf16 activations)
    bool round_bf16;      // f32 values rounded to bf16 (down input with bf16 activations)

    // values e0 .. e0 + 4*N - 1 (e0 a multiple of 4; of 8 for bf16 rows)
    template <int N>
    __device__ __forceinline__ void load(int e0, float (&v)[4 * N]) const
    {
        if (bf16_in) {
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) + e0);
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const uint4 r = src[i];
                const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    v[8 * i + 2 * q] = __uint_as_float(w[q] << 16);
                    v[8 * i + 2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
                }
            }
        } else {
            const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + e0);
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const float4 r = src[i];
                v[4 * i] = r.x;
                v[4 * i + 1] = r.y;
                v[4 * i + 2] = r.z;
                v[4 * i + 3] = r.w;
            }
            if (round_bf16)
#pragma unroll
                for (int i = 0; i < 4 * N; ++i) v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
        }
    }
};

// Build the records of `n` input rows into shared memory with all compute
// threads (tid < G2_NW * 32).  row_of(i) is row i's index in the input (x for
// gate/up, h for down).  `scr` holds G2_NW floats of scratch; `cb`/`ph` the
// compute barrier.  Returns false if a barrier wait gave up.
template <int WB, int NDIG, typename RowFn>
__device__ bool g2_build(const G2P &p, unsigned char *recs, int n, RowFn row_of, bool gateup, float *scr,
                         uint64_t *cb, uint32_t &ph, volatile int *abort_flag)
{
    using F = Fmt<WB>;
    constexpr int DW = F::DW, NQ = DW / 4, EPC = F::EPC;
    const int tid = threadIdx.x, nth = G2_NW * 32;
    const int K = p.K, cpr = p.cpr;
    const G2Rec RL = g2_rec(NDIG, K, cpr);
    const bool bf = p.afmt == QRX_A_BF16;
    for (int i = 0; i < n; ++i) {
        const int64_t row = row_of(i);
        unsigned char *rec = recs + (size_t)i * p.rec_bytes;
        G2Row src;
        src.bf16_in = gateup && bf;
        src.round_bf16 = !gateup && bf;
        src.base = src.bf16_in ? static_cast<const void *>(static_cast<const __nv_bfloat16 *>(p.x) + row * p.in_ld)
                               : static_cast<const void *>(static_cast<const float *>(p.x) + row * p.in_ld);
        if constexpr (NDIG == 3) {
            // the row's largest magnitude -> shift s (sigma = 2^-s); 8 values per load step
            float am = 0.f;
#pragma unroll 4
            for (int e = tid * 8; e < K; e += nth * 8) {
                float v[8];
                src.load<2>(e, v);
#pragma unroll
                for (int q = 0; q < 8; ++q) am = fmaxf(am, fabsf(v[q]));
            }
            am = warp_max(am);
            if ((tid & 31) == 0) scr[tid >> 5] = am;
            if (!g2_cbar(cb, ph, abort_flag)) return false;
            am = 0.f;
#pragma unroll
            for (int w = 0; w < G2_NW; ++w) am = fmaxf(am, scr[w]);
            const int sh = am != 0.f ? fixed_shift(am) : 0;
            const bool fast = sh >= -126 && sh <= 127;
            const float mul = fast ? __int_as_float((sh + 127) << 23) : 0.f;
            for (int c = tid; c < cpr; c += nth) {
                float v[EPC];
                src.load<EPC / 4>(c * EPC, v);
                uint32_t wd[3][DW];
                int cs0 = 0, cs1 = 0, cs2 = 0;       // the chunk's digit sums per plane
#pragma unroll
                for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                    for (int j = 0; j < F::UPW; ++j) {
                        uint32_t b0 = 0, b1 = 0, b2 = 0;
#pragma unroll
                        for (int by = 0; by < 4; ++by) {
                            const float x = v[elem_in_chunk<WB>(wi, j, by)];
                            int8_t d0 = 0, d1 = 0, d2 = 0;
                            if (am != 0.f) split3(__float2int_rn(fast ? __fmul_rn(x, mul) : ldexpf(x, sh)), d0, d1, d2);
                            b0 |= (uint32_t)(uint8_t)d0 << (8 * by);
                            b1 |= (uint32_t)(uint8_t)d1 << (8 * by);
                            b2 |= (uint32_t)(uint8_t)d2 << (8 * by);
                            cs0 += d0;
                            cs1 += d1;
                            cs2 += d2;
                        }
                        wd[0][wi * F::UPW + j] = b0;
                        wd[1][wi * F::UPW + j] = b1;
                        wd[2][wi * F::UPW + j] = b2;
                    }
#pragma unroll
                for (int pl = 0; pl < 3; ++pl)
#pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        *reinterpret_cast<uint4 *>(rec + ((size_t)(pl * NQ + q) * cpr + c) * 16) =
                            make_uint4(wd[pl][4 * q], wd[pl][4 * q + 1], wd[pl][4 * q + 2], wd[pl][4 * q + 3]);
                *reinterpret_cast<int4 *>(rec + RL.csum + (size_t)c * 16) = make_int4(cs0, cs1, cs2, 0);
            }
            if (tid == 0) {
                float sig = 0.f;
                if (am != 0.f) sig = (-sh >= -126 && -sh <= 127) ? __int_as_float((127 - sh) << 23) : ldexpf(1.f, -sh);
                *reinterpret_cast<float *>(rec + RL.hdr) = sig;
            }
            if (!g2_cbar(cb, ph, abort_flag)) return false;     // scr is reused by the next row
        } else {
            // Q8_0: codes and d_b per 32-block; a thread builds whole blocks
            // (int8: two chunks, int4: one chunk, int2: one chunk of two blocks)
            float *dsc = reinterpret_cast<float *>(rec + RL.hdr);
            int *cor = reinterpret_cast<int *>(rec + RL.hdr + (RL.bytes - RL.hdr) / 2);
            constexpr int EPU = EPC > 32 ? EPC : 32;            // elements per build unit
            for (int u0 = tid; u0 < K / EPU; u0 += nth) {
                int8_t code[EPU];
#pragma unroll
                for (int bb = 0; bb < EPU / 32; ++bb) {
                    const int b = u0 * (EPU / 32) + bb;
                    float dq = 0.f;
                    int csum = 0;
                    if (gateup && p.xq) {         // codes and scales from qrx_quantize_act_q8
                        const uint4 *qs = reinterpret_cast<const uint4 *>(p.xq + row * p.in_ld + b * 32);
                        const uint4 q0 = qs[0], q1 = qs[1];
                        const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                        for (int l = 0; l < 32; ++l) code[bb * 32 + l] = (int8_t)(w[l >> 2] >> (8 * (l & 3)));
                        dq = p.xd[row * (p.in_ld / 32) + b];
                    } else {                      // the same Q8_0 formula on the values
                        float v[32];
                        src.load<8>(b * 32, v);
                        float am = 0.f;
#pragma unroll
                        for (int l = 0; l < 32; ++l) am = fmaxf(am, fabsf(v[l]));
                        const float f = am != 0.f ? __fdiv_rn(127.f, am) : 0.f;
#pragma unroll
                        for (int l = 0; l < 32; ++l) code[bb * 32 + l] = (int8_t)(am != 0.f ? q8_code(v[l], f) : 0);
                        dq = am != 0.f ? __fdiv_rn(am, 127.f) : 0.f;
                    }
#pragma unroll
                    for (int l = 0; l < 32; ++l) csum += code[bb * 32 + l];
                    dsc[b] = dq;
                    cor[b] = -F::OFF * csum;
                }
#pragma unroll
                for (int cc = 0; cc < EPU / EPC; ++cc) {
                    const int c = u0 * (EPU / EPC) + cc;
                    uint32_t wd[DW];
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                        for (int j = 0; j < F::UPW; ++j) {
                            uint32_t bw = 0;
#pragma unroll
                            for (int by = 0; by < 4; ++by)
                                bw |= (uint32_t)(uint8_t)code[cc * EPC + elem_in_chunk<WB>(wi, j, by)] << (8 * by);
                            wd[wi * F::UPW + j] = bw;
                        }
#pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        *reinterpret_cast<uint4 *>(rec + ((size_t)q * cpr + c) * 16) =
                            make_uint4(wd[4 * q], wd[4 * q + 1], wd[4 * q + 2], wd[4 * q + 3]);
                }
            }
        }
    }
    return NDIG == 3 ? true : g2_cbar(cb, ph, abort_flag);
}

// ---------------------------------------------------------------- unit iterator
// The CTA's units in order: slot s, row blocks [u, uend) of it.
struct G2Units {
    const int64_t *pre;
    int nslots, nu, nrb;
    int64_t c0, c1;
    int s;
    int64_t u, uend;
    bool valid;
};

__device__ __forceinline__ int g2_slot_ntok(const G2P &p, int s, int nu)
{
    if (s < nu) {
        const int e = p.union_ids[s];
        return (e >= 0 && e < p.E) ? p.offsets[e + 1] - p.offsets[e] : 0;
    }
    return p.T;
}

// Cost of a unit: G2_BW for streaming its rows plus one per token (dot work).
constexpr int64_t G2_BW = 4;

__device__ void g2_units_next(G2Units &u)
{
    if (u.valid && ++u.u < u.uend) return;
    u.valid = false;
    for (;;) {
        u.s = u.s < 0 ? 0 : u.s + 1;
        if (u.s >= u.nslots || u.pre[u.s] >= u.c1) return;
        const int64_t cost = (u.pre[u.s + 1] - u.pre[u.s]) / u.nrb;
        if (cost <= 0) continue;
        const int64_t g0 = u.pre[u.s];
        int64_t bf = u.c0 > g0 ? (u.c0 - g0 + cost - 1) / cost : 0;
        int64_t be = u.c1 > g0 ? (u.c1 - g0 + cost - 1) / cost : 0;
        if (be > u.nrb) be = u.nrb;
        if (bf < be) {
            u.u = bf;
            u.uend = be;
            u.valid = true;
            return;
        }
    }
}

// ---------------------------------------------------------------- kernel
// Shared memory: the records, the compute barrier and flags, scratch, the
// slot cost prefix.
template <int WB, int NDIG, int TP, int R, bool GATEUP, bool PROBE>
__global__ void __launch_bounds__(G2_THREADS, 1) k_gemv2(const __grid_constant__ G2P p)
{
    using F = Fmt<WB>;
    constexpr int NM = GATEUP ? 2 : 1;
    constexpr int DW = F::DW, NQ = DW / 4, UPW = F::UPW;
    constexpr int NP = NDIG == 3 ? 3 : 1;                 // integer planes per (token, row)
    // int4: a packed word splits by one LOP3 per half -- the low nibbles as
    // they are, the high nibbles left in place (16 x the code) -- and the two
    // halves sum into separate exact accumulators, the second divided by 16
    constexpr bool HI16 = WB == 4;
    constexpr int NA = HI16 ? 2 : 1;
    constexpr int NBC = WB == 2 ? 2 : 1;                 // Q8_0 blocks a chunk touches
    constexpr int V = TP * NM * R;                        // values a lane reduces per unit
    extern __shared__ __align__(128) unsigned char sm[];
    uint64_t *cbar = reinterpret_cast<uint64_t *>(sm + p.bar_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(cbar + 1);
    int64_t *pre = reinterpret_cast<int64_t *>(sm + p.pre_off);
    float *scr = reinterpret_cast<float *>(sm + p.red_off);
    unsigned char *recs = sm + p.rec_off;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        mbar_init(g2_smem(cbar), G2_NW);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t cph = 0;      // barrier phase
    if constexpr (GATEUP) {
        // the records of every token, before the dependency wait: x is an input
        // of the call, so this overlaps the kernels that route
        if (!g2_build<WB, NDIG>(p, recs, p.T, [](int i) -> int64_t { return i; }, true, scr, cbar, cph, abort_flag))
            return;
    }
    pdl_wait();            // gate/up: the permutation; down: h, from the kernels before
    pdl_trigger();
    const int nu = p.routed ? *p.n_union : 0;
    const int nslots = nu + (p.shared ? 1 : 0);
    if (warp == 0) {       // cost prefix over slots
        int64_t run = 0;
        for (int s0 = 0; s0 < nslots; s0 += 32) {
            const int s = s0 + lane;
            int64_t cost = 0;
            if (s < nslots) {
                if (s < nu) {
                    const int e = p.union_ids[s];
                    if (e < 0 || e >= p.E) raise_status(DERR_BADIDX);
                }
                const int nt = g2_slot_ntok(p, s, nu);
                cost = nt > 0 ? (int64_t)p.nrb * (G2_BW + min(nt, TP)) : 0;
            }
            int64_t inc = cost;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (s < nslots) pre[s] = run + inc - cost;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pre[nslots] = run;
    }
    __syncthreads();
    const int64_t Ctot = pre[nslots];
    G2Units u;
    u.pre = pre;
    u.nslots = nslots;
    u.nu = nu;
    u.nrb = p.nrb;
    u.c0 = Ctot * blockIdx.x / gridDim.x;
    u.c1 = Ctot * (blockIdx.x + 1) / gridDim.x;
    u.s = -1;
    u.u = u.uend = 0;
    u.valid = false;
    g2_units_next(u);
    QRX_CHECK_ONLY(const int64_t n_pos = p.routed ? (int64_t)p.T * p.k : 0;)
    QRX_CHECK_ONLY(const int64_t n_out = max(n_pos, p.shared ? p.sh_out_row0 + p.T : (int64_t)0);)

    const int LPR = p.lpr, nj = p.nj;
    const int cl = lane % LPR, grp = lane / LPR;
    const int lrow0 = warp * p.rw + grp;              // this lane's row i is lrow0 + gpw * i (in the unit)
    const G2Rec RL = g2_rec(NDIG, p.K, p.cpr);
    // after the butterfly (V <= LPR) lane cl holds value cl / rep: that value's
    // token, row and (for gate/up: gate, with the up value on lane cl + rep)
    const int rep = V <= LPR ? LPR / V : 1;
    const int my_idx = cl / rep;
    const int my_t = my_idx / (NM * R), my_i = (my_idx / NM) % R;
    const bool writer = V <= LPR && cl % rep == 0 && (!GATEUP || (my_idx & 1) == 0);

    int cur_s = -1, nt = 0;
    int rec[TP];           // shared-memory offsets of the slot's token records
    int64_t orow[TP];
    int corr[TP][NP];      // NDIG = 3: OFF * (this lane's digit sums over its chunks), per plane
    float sig[TP];
#pragma unroll
    for (int t = 0; t < TP; ++t) {
        rec[t] = p.rec_off;
        orow[t] = 0;
        sig[t] = 1.f;
#pragma unroll
        for (int pl = 0; pl < NP; ++pl) corr[t][pl] = 0;
    }
    while (u.valid) {
        const bool routed = u.s < nu;
        int e = 0;
        if (routed) {
            e = p.union_ids[u.s];
            e = (e >= 0 && e < p.E) ? e : 0;
        }
        if (u.s != cur_s) {
            // ---- enter a slot: its tokens, their records, this lane's corrections
            const int p0 = routed ? p.offsets[e] : 0;
            nt = min(g2_slot_ntok(p, u.s, nu), TP);
            int64_t inrow[TP];
            bool ok = true;
#pragma unroll
            for (int i = 0; i < TP; ++i) {
                const int ii = min(i, max(nt - 1, 0));
                if (routed) {
                    QRX_CHECK_OR((int64_t)p0 + ii < n_pos, ok = false);
                    orow[i] = p0 + ii;
                    if constexpr (GATEUP) {
                        const int a = p.sorted[p0 + ii];
                        QRX_CHECK_OR(a >= 0 && a / p.k < p.T, ok = false);
                        inrow[i] = a / p.k;
                    } else {
                        inrow[i] = p0 + ii;
                    }
                } else {
                    orow[i] = p.sh_out_row0 + ii;
                    inrow[i] = GATEUP ? ii : p.sh_in_row0 + ii;
                }
            }
            if (!ok) return;
            if constexpr (GATEUP) {
#pragma unroll
                for (int i = 0; i < TP; ++i) rec[i] = p.rec_off + (int)inrow[i] * p.rec_bytes;
            } else {
                // every warp is done with the previous slot's records
                if (!g2_cbar(cbar, cph, abort_flag)) return;
                if (!g2_build<WB, NDIG>(p, recs, nt, [&](int i) -> int64_t { return g2_pick(inrow, i); }, false, scr,
                                        cbar, cph, abort_flag))
                    return;
#pragma unroll
                for (int i = 0; i < TP; ++i) rec[i] = p.rec_off + min(i, max(nt - 1, 0)) * p.rec_bytes;
            }
            if constexpr (NDIG == 3) {
#pragma unroll
                for (int t = 0; t < TP; ++t) {
                    sig[t] = *reinterpret_cast<const float *>(sm + rec[t] + RL.hdr);
                    int s0 = 0, s1 = 0, s2 = 0;
                    for (int j = 0; j < nj; ++j) {
                        const int4 c4 = *reinterpret_cast<const int4 *>(sm + rec[t] + RL.csum + (cl + LPR * j) * 16);
                        s0 += c4.x;
                        s1 += c4.y;
                        s2 += c4.z;
                    }
                    corr[t][0] = F::OFF * s0;
                    corr[t][1] = F::OFF * s1;
                    corr[t][2] = F::OFF * s2;
                }
            }
            cur_s = u.s;
        }
        // ---- one unit: this lane's rows, their row pointers and (writers) scales
        const int r0 = (int)(u.u * p.rb);
        const uint8_t *wrow[NM][R];
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const uint8_t *base = routed ? p.m[m].q + (int64_t)e * p.m[m].sq : p.msh[m].q;
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const int row = min(r0 + lrow0 + p.gpw * i, p.rows - 1);     // a row past the end is read, unused
                wrow[m][i] = base + (int64_t)row * p.row_bytes;
            }
        }
        float sc0 = 0.f, sc1 = 0.f;
        const int wr_row = r0 + lrow0 + p.gpw * my_i;
        if (writer && wr_row < p.rows) {
            sc0 = routed ? p.m[0].s[(int64_t)e * p.m[0].ss + wr_row] : p.msh[0].s[wr_row];
            if constexpr (GATEUP) sc1 = routed ? p.m[1].s[(int64_t)e * p.m[1].ss + wr_row] : p.msh[1].s[wr_row];
        }
        int iacc[TP][NM][R][NP][NA];
        float facc[TP][NM][R];
#pragma unroll
        for (int t = 0; t < TP; ++t)
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    facc[t][m][i] = 0.f;
#pragma unroll
                    for (int pl = 0; pl < NP; ++pl)
#pragma unroll
                        for (int h = 0; h < NA; ++h) iacc[t][m][i][pl][h] = 0;
                }
        auto load = [&](int j, uint4 (&b)[NM][R]) {
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int i = 0; i < R; ++i) b[m][i] = ld_stream16(wrow[m][i] + (size_t)(cl + LPR * j) * 16);
        };
        // chunk j of every row of this lane, against every token of the slot
        auto compute = [&](int j, const uint4 (&b)[NM][R]) {
            const int c = cl + LPR * j;
#pragma unroll
            for (int t = 0; t < TP; ++t) {
                if (t >= nt) break;
                const unsigned char *rt = sm + rec[t];
                const int cpr16 = p.cpr * 16;
                uint32_t d[NDIG][DW];
#pragma unroll
                for (int pl = 0; pl < NDIG; ++pl)
#pragma unroll
                    for (int q = 0; q < NQ; ++q) {
                        const uint4 d4 = *reinterpret_cast<const uint4 *>(rt + (pl * NQ + q) * cpr16 + c * 16);
                        d[pl][4 * q] = d4.x;
                        d[pl][4 * q + 1] = d4.y;
                        d[pl][4 * q + 2] = d4.z;
                        d[pl][4 * q + 3] = d4.w;
                    }
                float dq[NBC];
                int cb[NBC];
                if constexpr (NDIG == 1) {
                    const float *dsc = reinterpret_cast<const float *>(rt + RL.hdr);
                    const int *cor = reinterpret_cast<const int *>(rt + RL.hdr + (RL.bytes - RL.hdr) / 2);
#pragma unroll
                    for (int bc = 0; bc < NBC; ++bc) {
                        const int bb = WB == 8 ? (c >> 1) : (WB == 4 ? c : 2 * c + bc);
                        dq[bc] = dsc[bb];
                        cb[bc] = cor[bb];
                    }
                }
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        const uint32_t ww[4] = {b[m][i].x, b[m][i].y, b[m][i].z, b[m][i].w};
                        uint32_t uw[4][UPW];
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) {
                            if constexpr (HI16) {
                                uw[wi][0] = (ww[wi] ^ 0x88888888u) & 0x0F0F0F0Fu;   // elements 0, 2, 4, 6 (code + 8)
                                uw[wi][1] = (ww[wi] ^ 0x88888888u) & 0xF0F0F0F0u;   // elements 1, 3, 5, 7, x16
                            } else {
                                unpack_word<WB>(ww[wi], uw[wi]);
                            }
                        }
                        if constexpr (NDIG == 3) {
#pragma unroll
                            for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                                for (int jj = 0; jj < UPW; ++jj)
#pragma unroll
                                    for (int pl = 0; pl < 3; ++pl) {
                                        int &acc = iacc[t][m][i][pl][HI16 ? jj : 0];
                                        acc = HI16 ? g2_dp4a_us(uw[wi][jj], d[pl][wi * UPW + jj], acc)
                                                   : dp4a(uw[wi][jj], d[pl][wi * UPW + jj], acc);
                                    }
                        } else {
                            int ib[NBC], ibh = 0;
#pragma unroll
                            for (int bc = 0; bc < NBC; ++bc) ib[bc] = cb[bc];
#pragma unroll
                            for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                                for (int jj = 0; jj < UPW; ++jj) {
                                    const int bc = WB == 2 ? (wi >> 1) : 0;
                                    if (HI16 && jj == 1) ibh = g2_dp4a_us(uw[wi][jj], d[0][wi * UPW + jj], ibh);
                                    else ib[bc] = dp4a(uw[wi][jj], d[0][wi * UPW + jj], ib[bc]);
                                }
                            if constexpr (HI16) ib[0] += ibh >> 4;
                            // int8: a block is two chunks, on lanes 2b and 2b + 1
                            if constexpr (WB == 8) ib[0] += __shfl_xor_sync(0xffffffffu, ib[0], 1);
                            const bool mine = WB != 8 || (c & 1) == 0;
#pragma unroll
                            for (int bc = 0; bc < NBC; ++bc) {
                                if (mine) facc[t][m][i] = fmaf(dq[bc], (float)ib[bc], facc[t][m][i]);
                                if constexpr (PROBE) {
                                    const int64_t row = r0 + lrow0 + p.gpw * i;
                                    if (mine && row < p.rows) {
                                        const int bb = WB == 8 ? (c >> 1) : (WB == 4 ? c : 2 * c + bc);
                                        p.probe[((orow[t] * NM + m) * p.rows + row) * (int64_t)(p.K / 32) + bb] = ib[bc];
                                    }
                                }
                            }
                        }
                    }
            }
        };
        // the streaming loop: chunk j + 1's loads are issued before chunk j is computed
        uint4 bufA[NM][R], bufB[NM][R];
        load(0, bufA);
#pragma unroll 1
        for (int j = 0; j < nj; j += 2) {
            if (j + 1 < nj) load(j + 1, bufB);
            compute(j, bufA);
            if (j + 2 < nj) load(j + 2, bufA);
            if (j + 1 < nj) compute(j + 1, bufB);
        }
        // ---- epilogue: lane partials -> row totals -> scales -> outputs
        float v[V];
#pragma unroll
        for (int t = 0; t < TP; ++t)
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    float x;
                    if constexpr (NDIG == 3) {
                        int P[3];
#pragma unroll
                        for (int pl = 0; pl < 3; ++pl)
                            P[pl] = (HI16 ? iacc[t][m][i][pl][0] + (iacc[t][m][i][pl][NA - 1] >> 4) : iacc[t][m][i][pl][0]) -
                                    corr[t][pl];
                        x = fmaf(65536.f, (float)P[2], fmaf(256.f, (float)P[1], (float)P[0]));
                    }
                    else
                        x = facc[t][m][i];
                    v[(t * R + i) * NM + m] = t < nt ? x : 0.f;
                }
        if (LPR == 32) g2_tr_reduce<V, 32>(v, lane);
        else if (LPR == 16) g2_tr_reduce<V, 16>(v, lane);
        else if (LPR == 8) g2_tr_reduce<V, 8>(v, lane);
        else if (LPR == 4) g2_tr_reduce<V, 4>(v, lane);
        else if (LPR == 2) g2_tr_reduce<V, 2>(v, lane);
        // value idx's total tot (gate/up: and its up total upv) to the output
        auto emit = [&](int idx, float tot, float upv, float s0, float s1) {
            const int t = idx / (NM * R), i = (idx / NM) % R;
            const int row = r0 + lrow0 + p.gpw * i;
            if (t >= nt || row >= p.rows) return;
            const int64_t o = g2_pick(orow, t);
            QRX_CHECK_OR(o >= 0 && o < n_out, return);
            const float sg = NDIG == 3 ? g2_pick(sig, t) : 1.f;
            if constexpr (GATEUP)
                p.out[o * p.out_ld + row] = silu_mul(s0 * (sg * tot), s1 * (sg * upv));
            else
                p.out[o * p.out_ld + row] = s0 * (sg * tot);
        };
        if (V <= LPR) {
            const float upv = GATEUP ? __shfl_xor_sync(0xffffffffu, v[0], rep) : 0.f;
            if (writer) emit(my_idx, v[0], upv, sc0, sc1);
        } else {
            // few lanes per row (short rows): each lane holds V / LPR totals
            const int nv = V / LPR;
#pragma unroll
            for (int q = 0; q < V; q += NM) {
                if (q >= nv) break;
                const int idx = cl * nv + q;
                const int i = (idx / NM) % R;
                const int row = min(r0 + lrow0 + p.gpw * i, p.rows - 1);
                const float s0 = routed ? p.m[0].s[(int64_t)e * p.m[0].ss + row] : p.msh[0].s[row];
                const float s1 = GATEUP ? (routed ? p.m[NM - 1].s[(int64_t)e * p.m[NM - 1].ss + row] : p.msh[NM - 1].s[row]) : 0.f;
                emit(idx, v[q], GATEUP ? v[q + NM - 1] : 0.f, s0, s1);
            }
        }
        g2_units_next(u);
    }
}

// ---------------------------------------------------------------- host side
struct G2Plan {
    G2P p;
    int tp, r;
};

// Geometry for one projection: `nm` matrices of `rows` rows x K codes at wbits,
// activations with ndig digit planes, calls of T <= G2_TMAX tokens.  R (rows
// per lane per matrix) is 2 for gate/up and 4 for down: four row chunks per
// lane per step, double-buffered, keep ~64 KB of loads in flight per SM
// (halved for several tokens with f32 / bf16 digits, or int2, to fit the
// accumulators in registers).
static inline bool g2_plan(G2Plan &pl, int wbits, int ndig, int K, int rows, int nm, int T, int maxslots)
{
    G2P &p = pl.p;
    p = G2P{};
    if (T < 1 || T > G2_TMAX || rows < 1) return false;
    pl.tp = T == 1 ? 1 : (T == 2 ? 2 : 4);
    pl.r = nm == 2 ? 2 : 4;
    if (pl.tp >= 2 && (ndig == 3 || wbits == 2)) pl.r /= 2;   // several tokens' sums, or int2's wide unpack
    p.K = K;
    p.rows = rows;
    p.row_bytes = K * wbits / 8;
    if (p.row_bytes % 16) return false;
    p.cpr = p.row_bytes / 16;
    if (p.cpr >= 32) {
        if (p.cpr % 32) return false;
        p.lpr = 32;
        p.gpw = 1;
        p.nj = p.cpr / 32;
    } else {
        if (32 % p.cpr) return false;
        p.lpr = p.cpr;
        p.gpw = 32 / p.cpr;
        p.nj = 1;
    }
    p.rw = pl.r * p.gpw;
    p.rb = G2_NW * p.rw;
    p.nrb = (rows + p.rb - 1) / p.rb;
    p.rec_bytes = (g2_rec(ndig, K, p.cpr).bytes + 127) & ~127;
    p.nrec = nm == 2 ? T : pl.tp;               // gate/up: every token; down: one slot's rows
    int o = 0;
    p.rec_off = o;
    o += p.nrec * p.rec_bytes;
    p.bar_off = o;
    o += 16;
    p.red_off = o;
    o += 256;
    p.pre_off = o;
    o += (maxslots + 2) * 8;
    p.smem = o;
    return o <= G2_SMEM_MAX;
}

template <int WB, int ND, int TP, int R, bool GU, bool PR>
static cudaError_t g2_go(const G2P &p, int grid, cudaStream_t st)
{
    auto kern = k_gemv2<WB, ND, TP, R, GU, PR>;
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !(configured.load(std::memory_order_acquire) >> dev & 1ull)) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G2_SMEM_MAX);
        if (err != cudaSuccess) return err;
        if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
    }
    return launch_k(kern, dim3(grid), dim3(G2_THREADS), (size_t)p.smem, st, p);
}

template <bool GU, bool PR>
static cudaError_t g2_dispatch(const G2Plan &pl, int wbits, int ndig, int grid, cudaStream_t st)
{
    constexpr int R1 = GU ? 2 : 4, R2 = R1 / 2;     // rows per lane: one token; several (halved)
#define QRX_G2(WB, ND, TP, R) \
    if (wbits == WB && ndig == ND && pl.tp == TP && pl.r == R) return g2_go<WB, ND, TP, R, GU, PR>(pl.p, grid, st);
    if constexpr (PR) {        // Q8_0 with the block-sum side output
        QRX_G2(4, 1, 1, R1) QRX_G2(4, 1, 2, R1) QRX_G2(4, 1, 4, R1)
        QRX_G2(8, 1, 1, R1) QRX_G2(8, 1, 2, R1) QRX_G2(8, 1, 4, R1)
        QRX_G2(2, 1, 1, R1) QRX_G2(2, 1, 2, R2) QRX_G2(2, 1, 4, R2)
    } else {
        QRX_G2(4, 3, 1, R1) QRX_G2(4, 3, 2, R2) QRX_G2(4, 3, 4, R2) QRX_G2(4, 1, 1, R1) QRX_G2(4, 1, 2, R1) QRX_G2(4, 1, 4, R1)
        QRX_G2(8, 3, 1, R1) QRX_G2(8, 3, 2, R2) QRX_G2(8, 3, 4, R2) QRX_G2(8, 1, 1, R1) QRX_G2(8, 1, 2, R1) QRX_G2(8, 1, 4, R1)
        QRX_G2(2, 3, 1, R1) QRX_G2(2, 3, 2, R2) QRX_G2(2, 3, 4, R2) QRX_G2(2, 1, 1, R1) QRX_G2(2, 1, 2, R2) QRX_G2(2, 1, 4, R2)
    }
#undef QRX_G2
    return cudaErrorInvalidValue;
}

static inline void g2_common(G2P &p, const FfnArgs &a)
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

static inline G2Mat g2_mat(const MatRef &m) { return G2Mat{m.q, m.s, m.sq, m.ss}; }

bool g2_use(const FfnArgs &a)
{
    if (a.T < 1 || a.T > G2_TMAX) return false;
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    G2Plan pg, pd;
    return g2_plan(pg, a.wbits, ndig, a.H, a.I, 2, a.T, a.E + 1) && g2_plan(pd, a.wbits, ndig, a.I, a.H, 1, a.T, a.E + 1);
}

cudaError_t launch_g2_gateup(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    G2Plan pl;
    if (!g2_plan(pl, a.wbits, ndig, a.H, a.I, 2, a.T, a.E + 1)) return cudaErrorInvalidValue;
    G2P &p = pl.p;
    g2_common(p, a);
    p.m[0] = g2_mat(a.gate);
    p.m[1] = g2_mat(a.up);
    p.msh[0] = g2_mat(a.gate_sh);
    p.msh[1] = g2_mat(a.up_sh);
    p.x = a.x;
    p.xq = a.xq;
    p.xd = a.xd;
    p.in_ld = a.H;
    p.sh_in_row0 = 0;
    p.out = a.h;
    p.out_ld = a.h_ld;
    p.sh_out_row0 = a.sh_h_row0;
    p.probe = probe;
    if (probe) return ndig == 1 ? g2_dispatch<true, true>(pl, a.wbits, ndig, num_sms, st) : cudaErrorInvalidValue;
    return g2_dispatch<true, false>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_g2_down(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = a.afmt == QRX_A_Q8_0 ? 1 : 3;
    G2Plan pl;
    if (!g2_plan(pl, a.wbits, ndig, a.I, a.H, 1, a.T, a.E + 1)) return cudaErrorInvalidValue;
    G2P &p = pl.p;
    g2_common(p, a);
    p.m[0] = p.m[1] = g2_mat(a.down);
    p.msh[0] = p.msh[1] = g2_mat(a.down_sh);
    p.x = a.h;
    p.xq = nullptr;
    p.xd = nullptr;
    p.in_ld = a.h_ld;
    p.sh_in_row0 = a.sh_h_row0;
    p.out = a.y;
    p.out_ld = a.y_ld;
    p.sh_out_row0 = a.sh_y_row0;
    p.probe = probe;
    if (probe) return ndig == 1 ? g2_dispatch<false, true>(pl, a.wbits, ndig, num_sms, st) : cudaErrorInvalidValue;
    return g2_dispatch<false, false>(pl, a.wbits, ndig, num_sms, st);
}

}  // namespace qrx
