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
// Work.  A slot is one expert of the union (or the shared expert) with its
// tokens.  A warp-unit is (slot, group of RW consecutive rows): for gate/up
// the RW gate rows and the same RW up rows, so the SwiGLU is applied where
// both sums meet.  The warp-units of all slots are cut into contiguous ranges
// of equal estimated cost, one range per CTA (one CTA of 16 warps per SM), and
// a CTA's range into 16 contiguous runs, one per warp.  Warps never wait for
// one another while they stream.
//
// A warp streams its rows for the whole of K: lane l reads 16-byte chunks l,
// l + 32, ... of each row straight from HBM (128-bit loads that skip L1, the
// next chunk's loads issued before the current chunk is computed), unpacks
// the codes in registers and dots them with the activation digits (dp4a); its
// integer sums run over all of K, and the warp-unit ends with one transposed
// warp butterfly and the epilogue (row scales, SwiGLU).  Rows of fewer than 32
// chunks are covered by LPR = chunks lanes each, several rows per warp.
//
// Activations.  Every input row (a token of x for gate/up, a row of h for
// down) is turned into a "record" in shared memory by the whole CTA: NDIG
// digit planes of signed bytes in the order the unpacked weight words use, so
// each dot of 4 codes by 4 digits is one dp4a with an exact int32 sum.
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
//
// Fused steps of the layer forward.  With `fuse` set, every gate/up CTA first
// makes the router's choice and the batch-union permutation of the call's
// tokens itself, from the router logits (the same arithmetic as the selection
// and permutation kernels, so the same results), and CTA 0 publishes them
// (top-k indices and weights, the permutation, a compact slot table for the
// down projection).  With `comb` set, the down projection also applies the
// weighted combine: the warp that writes the last slot's rows of a row group
// (a per-group counter, zeroed by the fused gate/up) adds that group's rows
// over the token's experts, in ascending j, onto the shared expert's rows.
#pragma once
#include "qrx_dev.cuh"
#include "qrx_check.cuh"

namespace qrx {

constexpr int G2_NW = 16;                         // warps per CTA
constexpr int G2_THREADS = 32 * G2_NW;
constexpr int G2_TMAX = 4;                        // tokens per call
constexpr int G2_SMEM_MAX = 227 * 1024;
constexpr int G2_CLIST = 1024;                    // combine: row groups a CTA lists in shared memory
constexpr int64_t G2_BW = 4;                      // cost of a warp-unit: G2_BW for its bytes, plus one per token

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

// Compact slot table in global memory (written by the fused gate/up, read by
// the down projection): [0] slots (routed + shared), [1] routed slots, then
// per slot s ints 4 + 4s .. 4s + 7: expert (-1: shared), first position,
// tokens, 0.
constexpr int G2_TAB_HDR = 4;

struct G2P {
    int K, rows, row_bytes, cpr;     // codes per input row, rows per matrix, bytes per row, chunks per row
    int lpr, gpw, nj;                // lanes per row, row groups per warp, chunks per lane per row
    int rw, nwu;                     // rows per warp-unit (per matrix), warp-units per slot
    int rec_bytes, nrec, slot_cap;   // record size, records held, slots per phase (down)
    int ntile;                       // multi-token kernel: bytes of a warp's tile ring
    int allrec;                      // multi-token gate/up: one record per token of the call, built once
    int ms;                          // slot capacity of the tables (routed slots + 1)
    // shared-memory offsets (bytes)
    int o_sl, o_srt, o_pre, o_seg, o_hmx, o_rmax, o_route, o_rec, smem;
    G2Mat m[2], msh[2];              // gate/up: m[0] gate, m[1] up; down: m[0] down
    int routed, shared;
    int32_t *counts, *offsets, *sorted, *inv, *union_ids, *n_union;   // the permutation
    const int32_t *tab;              // down: compact slot table (null: from the permutation)
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
    // fused selection and permutation (gate/up)
    int fuse;
    const float *logits, *bias;      // [T][E], [E]
    int G, Gk;
    float rsf;
    double topp_thr;                 // 0: off
    int32_t *idx;                    // [T][k] outputs
    float *w;
    uint64_t *usage;                 // per-expert counters (may be null)
    int32_t *tab_out;                // the compact slot table
    int32_t *cnt;                    // combine counters to zero (fuse) / to count on (comb)
    int ncnt;
    // fused combine (down)
    int comb;
    const float *cw;                 // [T][k] weights
    const int32_t *cinv;             // [T][k] positions (-1: none)
    float *cout;                     // [T][H]
    // largest |h| per h row, as f32 bits (fused path; zeroed before the gate/up
    // launch): gate/up raises it for every h value it writes, down reads it
    uint32_t *hmax;
};

// ---------------------------------------------------------------- small helpers
// dp4a of unsigned weight bytes by signed digit bytes: int4 high halves are
// kept in place (16 x the code), which needs the unsigned form.
__device__ __forceinline__ int g2_dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
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

// A team of consecutive warps of the CTA that works and synchronises on its
// own (named barrier `bar`; bar 0 with every thread is __syncthreads).
struct G2Team {
    int tid, nthr, warp, nwarp, bar;
    __device__ void sync() const { asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nthr) : "memory"); }
};
__device__ __forceinline__ G2Team g2_cta()
{
    return G2Team{(int)threadIdx.x, G2_THREADS, (int)(threadIdx.x >> 5), G2_NW, 0};
}

// ---------------------------------------------------------------- record builder
// EW consecutive values e0 .. e0 + EW - 1 of one input row as the dot sees
// them (EW = 4, 8 or 16; e0 a multiple of EW): f32 rows (x, or h -- rounded to
// bf16 first for bf16 activations) or bf16 rows (x).
template <int EW>
__device__ __forceinline__ void g2_vals(const void *row, bool bf16_in, bool round_bf16, int e0, float (&v)[EW])
{
    if (bf16_in) {
        const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(row) + e0;
        uint32_t wd[EW / 2];
        if constexpr (EW == 4) {
            const uint2 r = __ldg(reinterpret_cast<const uint2 *>(src));
            wd[0] = r.x;
            wd[1] = r.y;
        } else {
#pragma unroll
            for (int i = 0; i < EW / 8; ++i) {
                const uint4 r = __ldg(reinterpret_cast<const uint4 *>(src) + i);
                wd[4 * i] = r.x;
                wd[4 * i + 1] = r.y;
                wd[4 * i + 2] = r.z;
                wd[4 * i + 3] = r.w;
            }
        }
#pragma unroll
        for (int q = 0; q < EW / 2; ++q) {
            v[2 * q] = __uint_as_float(wd[q] << 16);
            v[2 * q + 1] = __uint_as_float(wd[q] & 0xFFFF0000u);
        }
    } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(row) + e0);
#pragma unroll
        for (int i = 0; i < EW / 4; ++i) {
            const float4 r = __ldg(src + i);
            v[4 * i] = r.x;
            v[4 * i + 1] = r.y;
            v[4 * i + 2] = r.z;
            v[4 * i + 3] = r.w;
        }
        if (round_bf16)
#pragma unroll
            for (int i = 0; i < EW; ++i) v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    }
}

// Store the UPW digit words of packed word wi of chunk c (one plane) into a record.
template <int WB>
__device__ __forceinline__ void g2_put_words(unsigned char *plane, int cpr, int c, int wi, const uint32_t (&wd)[Fmt<WB>::UPW])
{
    constexpr int UPW = Fmt<WB>::UPW;
    if constexpr (UPW == 1) {
        *reinterpret_cast<uint32_t *>(plane + (size_t)c * 16 + wi * 4) = wd[0];
    } else if constexpr (UPW == 2) {
        *reinterpret_cast<uint2 *>(plane + ((size_t)(wi >> 1) * cpr + c) * 16 + (wi & 1) * 8) = make_uint2(wd[0], wd[1]);
    } else {
        *reinterpret_cast<uint4 *>(plane + ((size_t)wi * cpr + c) * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
}

// Build the records of n input rows with the whole CTA.  An item is one packed
// weight word's worth of elements (EW = EPC / 4 values): item it covers chunk
// it / 4, word it % 4, so the four items of a chunk sit on four neighbouring
// lanes.  src(i, row) gives record i's input row (false: record i is unused).
// rmax: n * G2_NW floats of scratch.  Ends with __syncthreads.
template <int WB, int NDIG, bool CACHE, typename SrcFn>
__device__ void g2_build(const G2P &p, unsigned char *recs, int n, SrcFn src, bool gateup, float *rmax,
                         const G2Team tm = g2_cta())
{
    using F = Fmt<WB>;
    constexpr int EW = F::EPC / 4, UPW = F::UPW, NQ = F::DW / 4;
    const int tid = tm.tid, lane = threadIdx.x & 31, warp = tm.warp, NTH = tm.nthr;
    const int K = p.K, cpr = p.cpr, nitem = K / EW;
    const G2Rec RL = g2_rec(NDIG, K, cpr);
    const bool bf_in = gateup && p.afmt == QRX_A_BF16, rnd = !gateup && p.afmt == QRX_A_BF16;
    auto row_ptr = [&](int64_t row) -> const void * {
        return bf_in ? static_cast<const void *>(static_cast<const __nv_bfloat16 *>(p.x) + row * p.in_ld)
                     : static_cast<const void *>(static_cast<const float *>(p.x) + row * p.in_ld);
    };
    if constexpr (NDIG == 3) {
        // the row maxima of h are known (fused down projection): one pass
        const bool known = !gateup && p.hmax != nullptr;
        // pass 1: every row's largest magnitude; a thread's first two (row, item)
        // values stay in registers for pass 2 (item it = tid + q * threads in both)
        const int nq = (nitem + NTH - 1) / NTH;
        float cache[2][EW];
        for (int i = 0; i < n && !known; ++i) {
            int64_t row;
            if (!src(i, row)) continue;
            const void *rp = row_ptr(row);
            float am = 0.f;
            for (int it = tid, q = 0; it < nitem; it += NTH, ++q) {
                float v[EW];
                g2_vals<EW>(rp, bf_in, rnd, it * EW, v);
                const int slot = i * nq + q;
#pragma unroll
                for (int e = 0; e < EW; ++e) {
                    am = fmaxf(am, fabsf(v[e]));
                    if (CACHE && slot == 0) cache[0][e] = v[e];
                    if (CACHE && slot == 1) cache[1][e] = v[e];
                }
            }
            am = warp_max(am);
            if (lane == 0) rmax[i * G2_NW + warp] = am;
        }
        if (!known) tm.sync();
        // pass 2: digits and chunk digit sums
        for (int i = 0; i < n; ++i) {
            int64_t row;
            if (!src(i, row)) continue;
            const void *rp = row_ptr(row);
            unsigned char *rec = recs + (size_t)i * p.rec_bytes;
            float am = 0.f;
            if (known) {
                am = __uint_as_float(p.hmax[row]);
                if (rnd) am = __bfloat162float(__float2bfloat16_rn(am));
            } else {
                for (int w = 0; w < tm.nwarp; ++w) am = fmaxf(am, rmax[i * G2_NW + w]);
            }
            const int sh = am != 0.f ? fixed_shift(am) : 0;
            const bool fast = sh >= -126 && sh <= 127;
            const float mul = fast ? __int_as_float((sh + 127) << 23) : 0.f;
            for (int base = warp * 32, q = 0; base < nitem; base += NTH, ++q) {
                const int it = base + lane;
                const bool act = it < nitem;
                const int c = it >> 2, wi = it & 3, slot = i * nq + q;
                float v[EW];
                if (act && (!CACHE || known || slot >= 2)) g2_vals<EW>(rp, bf_in, rnd, it * EW, v);
                else
#pragma unroll
                    for (int e = 0; e < EW; ++e) v[e] = !act ? 0.f : slot == 0 ? cache[0][e] : cache[1][e];
                uint32_t wd[3][UPW];
                int cs0 = 0, cs1 = 0, cs2 = 0;
#pragma unroll
                for (int j = 0; j < UPW; ++j) {
                    uint32_t b0 = 0, b1 = 0, b2 = 0;
#pragma unroll
                    for (int by = 0; by < 4; ++by) {
                        const float x = v[elem_in_chunk<WB>(0, j, by)];
                        int8_t d0 = 0, d1 = 0, d2 = 0;
                        if (am != 0.f) split3(__float2int_rn(fast ? __fmul_rn(x, mul) : ldexpf(x, sh)), d0, d1, d2);
                        b0 |= (uint32_t)(uint8_t)d0 << (8 * by);
                        b1 |= (uint32_t)(uint8_t)d1 << (8 * by);
                        b2 |= (uint32_t)(uint8_t)d2 << (8 * by);
                        cs0 += d0;
                        cs1 += d1;
                        cs2 += d2;
                    }
                    wd[0][j] = b0;
                    wd[1][j] = b1;
                    wd[2][j] = b2;
                }
#pragma unroll
                for (int o = 1; o < 4; o <<= 1) {
                    cs0 += __shfl_xor_sync(0xffffffffu, cs0, o);
                    cs1 += __shfl_xor_sync(0xffffffffu, cs1, o);
                    cs2 += __shfl_xor_sync(0xffffffffu, cs2, o);
                }
                if (act) {
#pragma unroll
                    for (int pl = 0; pl < 3; ++pl)
                        g2_put_words<WB>(rec + (size_t)pl * NQ * cpr * 16, cpr, c, wi, wd[pl]);
                    if (wi == 0) *reinterpret_cast<int4 *>(rec + RL.csum + (size_t)c * 16) = make_int4(cs0, cs1, cs2, 0);
                }
            }
            if (tid == 0) {
                float sig = 0.f;
                if (am != 0.f) sig = (-sh >= -126 && -sh <= 127) ? __int_as_float((127 - sh) << 23) : ldexpf(1.f, -sh);
                *reinterpret_cast<float *>(rec + RL.hdr) = sig;
            }
        }
    } else {
        // Q8_0: codes and d_b per 32-block, IPB items per block on neighbouring lanes
        constexpr int IPB = 32 / EW;
        for (int i = 0; i < n; ++i) {
            int64_t row;
            if (!src(i, row)) continue;
            const void *rp = row_ptr(row);
            unsigned char *rec = recs + (size_t)i * p.rec_bytes;
            float *dsc = reinterpret_cast<float *>(rec + RL.hdr);
            int *cor = reinterpret_cast<int *>(rec + RL.hdr + (RL.bytes - RL.hdr) / 2);
            for (int base = warp * 32; base < nitem; base += NTH) {
                const int it = base + lane;
                const bool act = it < nitem;
                const int c = it >> 2, wi = it & 3, b = it / IPB;
                int code[EW];
                float dq = 0.f;
                if (gateup && p.xq) {         // codes and scales from qrx_quantize_act_q8
                    const int8_t *qs = p.xq + row * p.in_ld + (int64_t)it * EW;
                    uint32_t qw[EW / 4];
                    if (act) {
                        if constexpr (EW == 4) {
                            qw[0] = *reinterpret_cast<const uint32_t *>(qs);
                        } else if constexpr (EW == 8) {
                            const uint2 r = *reinterpret_cast<const uint2 *>(qs);
                            qw[0] = r.x;
                            qw[1] = r.y;
                        } else {
                            const uint4 r = *reinterpret_cast<const uint4 *>(qs);
                            qw[0] = r.x;
                            qw[1] = r.y;
                            qw[2] = r.z;
                            qw[3] = r.w;
                        }
                        dq = p.xd[row * (p.in_ld / 32) + b];
                    } else {
#pragma unroll
                        for (int q = 0; q < EW / 4; ++q) qw[q] = 0;
                    }
#pragma unroll
                    for (int l = 0; l < EW; ++l) code[l] = (int8_t)(qw[l >> 2] >> (8 * (l & 3)));
                } else {                      // the same Q8_0 formula on the values
                    float v[EW];
                    if (act) g2_vals<EW>(rp, bf_in, rnd, it * EW, v);
                    else
#pragma unroll
                        for (int q = 0; q < EW; ++q) v[q] = 0.f;
                    float am = 0.f;
#pragma unroll
                    for (int l = 0; l < EW; ++l) am = fmaxf(am, fabsf(v[l]));
#pragma unroll
                    for (int o = 1; o < IPB; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
                    const float f = am != 0.f ? __fdiv_rn(127.f, am) : 0.f;
#pragma unroll
                    for (int l = 0; l < EW; ++l) code[l] = am != 0.f ? q8_code(v[l], f) : 0;
                    dq = am != 0.f ? __fdiv_rn(am, 127.f) : 0.f;
                }
                int csum = 0;
#pragma unroll
                for (int l = 0; l < EW; ++l) csum += code[l];
#pragma unroll
                for (int o = 1; o < IPB; o <<= 1) csum += __shfl_xor_sync(0xffffffffu, csum, o);
                uint32_t wd[UPW];
#pragma unroll
                for (int j = 0; j < UPW; ++j) {
                    uint32_t bw = 0;
#pragma unroll
                    for (int by = 0; by < 4; ++by) bw |= (uint32_t)(uint8_t)code[elem_in_chunk<WB>(0, j, by)] << (8 * by);
                    wd[j] = bw;
                }
                if (act) {
                    g2_put_words<WB>(rec, cpr, c, wi, wd);
                    if (it % IPB == 0) {
                        dsc[b] = dq;
                        cor[b] = -F::OFF * csum;
                    }
                }
            }
        }
    }
    tm.sync();
}

// ---------------------------------------------------------------- slot tables
// Shared-memory slot table: [0] slots, [1] routed slots, then expert, first
// position and token count per slot (arrays of p.ms ints from int 4 on).
struct G2Slots {
    int *hdr, *e, *p0, *nt;
    __device__ G2Slots(int *base, int ms) : hdr(base), e(base + 4), p0(base + 4 + ms), nt(base + 4 + 2 * ms) {}
};

// Route scratch in shared memory, for T tokens, E experts, G groups, top-k.
struct G2RouteSm {
    float *s, *sc, *csc, *gsc;
    int *kg, *cand, *pick, *ridx, *pos, *lead, *less, *cnt;
    float *rw;
    __host__ __device__ static int ints(int T, int E, int G, int Gk, int k)
    {
        const int A = T * k;
        return 4 * T * E + T * G + T * Gk + T * k + 6 * A;
    }
    __device__ G2RouteSm(int *b, int T, int E, int G, int Gk, int k)
    {
        const int A = T * k;
        s = reinterpret_cast<float *>(b);
        sc = s + T * E;
        csc = sc + T * E;
        cand = reinterpret_cast<int *>(csc + T * E);
        gsc = reinterpret_cast<float *>(cand + T * E);
        kg = reinterpret_cast<int *>(gsc + T * G);
        pick = kg + T * Gk;
        ridx = pick + T * k;
        rw = reinterpret_cast<float *>(ridx + A);
        pos = reinterpret_cast<int *>(rw + A);
        lead = pos + A;
        less = lead + A;
        cnt = less + A;
    }
};

// CTA 0 publishes the route: choice, permutation, usage, the compact slot
// table; and zeroes the combine counters.  Every thread of the CTA calls it.
__device__ void g2_publish(const G2P &p, const G2RouteSm &r, G2Slots sl, int A, int nu, int nslots,
                           const G2Team tm = g2_cta())
{
    const int tid = tm.tid, E = p.E, NTH = tm.nthr;
    {
        for (int a = tid; a < A; a += NTH) {
            p.idx[a] = r.ridx[a];
            p.w[a] = r.rw[a];
            p.inv[a] = r.pos[a];
            if (r.pos[a] >= 0) p.sorted[r.pos[a]] = a;
            if (r.lead[a] && p.usage)
                atomicAdd(reinterpret_cast<unsigned long long *>(p.usage + r.ridx[a]), (unsigned long long)r.cnt[a]);
        }
        for (int e = tid; e <= E; e += NTH) {
            int less = 0, cnt = 0;
            for (int b = 0; b < A; ++b) {
                const int f = r.ridx[b];
                if (f < 0) continue;
                less += f < e;
                cnt += f == e;
            }
            p.offsets[e] = less;
            if (e < E) p.counts[e] = cnt;
        }
        for (int u = tid; u < nu; u += NTH) p.union_ids[u] = sl.e[u];
        for (int s = tid; s < nslots; s += NTH) {
            p.tab_out[G2_TAB_HDR + 4 * s] = sl.e[s];
            p.tab_out[G2_TAB_HDR + 4 * s + 1] = sl.p0[s];
            p.tab_out[G2_TAB_HDR + 4 * s + 2] = sl.nt[s];
            p.tab_out[G2_TAB_HDR + 4 * s + 3] = 0;
        }
        if (tid == 0) {
            *p.n_union = nu;
            p.tab_out[0] = nslots;
            p.tab_out[1] = nu;
            p.tab_out[2] = 0;
            p.tab_out[3] = 0;
        }
        for (int i = tid; i < p.ncnt; i += NTH) p.cnt[i] = 0;
    }
}

// The call's expert choice and batch-union permutation, made by every CTA in
// shared memory.  Selection (README "JustVugg/colibri", section "已实现的功能":
// DeepSeek-V3-style sigmoid router, noaux_tc): s = sigmoid(logit) in double
// rounded to f32, biased score sc = s + bias (selection only); a group's score
// is the sum of its two largest sc; the Gk best groups are kept (ties to the
// lower group); the k largest sc among their experts are chosen (ties to the
// lower expert), in descending order; weights are s_j / sum(s) * rsf with the
// sum in double in that order; then adaptive top-p when on.  Permutation: a
// stable counting sort of the assignments a = t*k + j by expert (dropped ones,
// -1, take no position).  CTA 0 writes the results to memory.  Ends with
// __syncthreads; fills the slot table (routed slots in ascending expert, then
// the shared slot) and srt (position -> assignment).
__device__ void g2_route(const G2P &p, int *rsm, G2Slots sl, int *srt)
{
    const int T = p.T, E = p.E, G = p.G, Gk = p.Gk, k = p.k, gs = E / G, A = T * k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    G2RouteSm r(rsm, T, E, G, Gk, k);
    // sigmoid and biased scores
    for (int i = tid; i < T * E; i += G2_THREADS) {
        const float lg = p.logits[i];
        const float s = (float)(1.0 / (1.0 + exp(-(double)lg)));
        r.s[i] = s;
        r.sc[i] = __fadd_rn(s, p.bias[i % E]);
    }
    __syncthreads();
    // group scores: top-2 sum per (token, group), one warp each
    for (int q = warp; q < T * G; q += G2_NW) {
        const int t = q / G, g = q % G;
        float t1 = -INFINITY, t2 = -INFINITY;
        for (int e = g * gs + lane; e < (g + 1) * gs; e += 32) {
            const float v = r.sc[t * E + e];
            if (v > t1) { t2 = t1; t1 = v; }
            else if (v > t2) { t2 = v; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float b1 = __shfl_xor_sync(0xffffffffu, t1, o), b2 = __shfl_xor_sync(0xffffffffu, t2, o);
            const float hi = fmaxf(t1, b1), lo = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
            t1 = hi;
            t2 = lo;
        }
        if (lane == 0) r.gsc[q] = gs >= 2 ? __fadd_rn(t1, t2) : t1;
    }
    __syncthreads();
    // kept groups (rank among the G scores, ties to the lower group), listed
    // in ascending group order: kg[t][i] = the i-th kept group
    for (int q = tid; q < T * G; q += G2_THREADS) {
        const int t = q / G, g = q % G;
        const float *gt = r.gsc + t * G;
        int before = 0;
        bool kept = false;
        for (int g2 = 0; g2 <= g; ++g2) {
            const float v = gt[g2];
            int rank = 0;
            for (int h = 0; h < G; ++h) {
                const float u = gt[h];
                rank += (u > v) || (u == v && h < g2);
            }
            if (g2 < g) before += rank < Gk;
            else kept = rank < Gk;
        }
        if (kept) r.kg[t * Gk + before] = g;
    }
    __syncthreads();
    // candidates (the kept groups' experts, ascending) and their biased scores, contiguous
    const int nc = Gk * gs;
    for (int q = tid; q < T * nc; q += G2_THREADS) {
        const int t = q / nc, c = q % nc;
        const int e = r.kg[t * Gk + c / gs] * gs + c % gs;
        r.cand[t * E + c] = e;
        r.csc[t * E + c] = r.sc[t * E + e];
    }
    __syncthreads();
    // picks: a candidate's rank by (sc descending, expert ascending); the
    // candidates are in ascending expert order, so a lower expert is a lower c
    for (int q = tid; q < T * nc; q += G2_THREADS) {
        const int t = q / nc, c = q % nc;
        const float *ct = r.csc + t * E;
        const float v = ct[c];
        int rank = 0;
#pragma unroll 8
        for (int c2 = 0; c2 < nc; ++c2) {
            const float u = ct[c2];
            rank += (u > v) || (u == v && c2 < c);
        }
        if (rank < k) r.pick[t * k + rank] = r.cand[t * E + c];
    }
    __syncthreads();
    // weights (warp t), top-p
    if (warp < T) {
        const int t = warp;
        double ssum = 0.0;
        for (int j = 0; j < k; ++j) ssum += (double)r.s[t * E + r.pick[t * k + j]];
        const int e = lane < k ? r.pick[t * k + lane] : 0;
        const float wv = lane < k ? (float)((double)r.s[t * E + e] / ssum * (double)p.rsf) : 0.f;
        const bool keep = p.topp_thr > 0.0 ? warp_topp_keep(lane, k, wv, p.topp_thr) : true;
        if (lane < k) {
            r.ridx[t * k + lane] = keep ? e : -1;
            r.rw[t * k + lane] = keep ? wv : 0.f;
        }
    }
    __syncthreads();
    // permutation: position = assignments of lower experts + earlier ones of the same
    for (int a = tid; a < A; a += G2_THREADS) {
        const int e = r.ridx[a];
        int less = 0, bef = 0, cnt = 0;
        for (int b = 0; b < A; ++b) {
            const int f = r.ridx[b];
            if (f < 0) continue;
            less += f < e;
            bef += (f == e) && (b < a);
            cnt += f == e;
        }
        const bool valid = e >= 0;
        r.pos[a] = valid ? less + bef : -1;
        r.lead[a] = valid && bef == 0;
        r.less[a] = less;
        r.cnt[a] = cnt;
        if (valid) srt[less + bef] = a;
    }
    __syncthreads();
    for (int a = tid; a < A; a += G2_THREADS) {
        if (!r.lead[a]) continue;
        const int e = r.ridx[a];
        int u = 0;
        for (int b = 0; b < A; ++b) u += r.lead[b] && r.ridx[b] < e;
        sl.e[u] = e;
        sl.p0[u] = r.less[a];
        sl.nt[u] = r.cnt[a];
    }
    int nu = 0;
    for (int b = 0; b < A; ++b) nu += r.lead[b];
    const int nslots = nu + (p.shared ? 1 : 0);
    if (tid == 0) {
        sl.hdr[0] = nslots;
        sl.hdr[1] = nu;
        if (p.shared) {
            sl.e[nu] = -1;
            sl.p0[nu] = 0;
            sl.nt[nu] = T;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) g2_publish(p, r, sl, A, nu, nslots);
}

// One token, groups of a multiple of 32 experts: the choice in four CTA steps
// (the same arithmetic and ties as g2_route).  (1) s and the biased scores sc
// of every expert; (2) one warp per group: the top-2 sum by a butterfly;
// (3) every expert of a kept group (rank of its group < Gk, ties to the lower
// group) counts, over the kept groups' experts, those with a larger sc or an
// equal sc and a lower index -- two threads per expert, half the members
// each -- and if the count is below k it is the pick of that rank; (4) warp 0:
// the weight sum in double in pick order, the weights, top-p, and the sort of
// the kept picks into the slot table.  CTA 0 publishes.  Ends with __syncthreads.
__host__ __device__ inline bool g2_route1_ok(int T, int E, int G, int k)
{
    return T == 1 && G >= 1 && G <= 32 && E % G == 0 && (E / G) % 32 == 0 && k <= 32;
}

__device__ void g2_route1(const G2P &p, int *rsm, G2Slots sl, int *srt, const G2Team tm = g2_cta())
{
    const int E = p.E, G = p.G, Gk = p.Gk, k = p.k, gs = E / G;
    const int tid = tm.tid, lane = threadIdx.x & 31, warp = tm.warp;
    G2RouteSm r(rsm, 1, E, G, Gk, k);
    float *ps = r.csc;                        // s of the pick of each rank
    for (int e = tid; e < E; e += tm.nthr) {
        const float s = (float)(1.0 / (1.0 + exp(-(double)p.logits[e])));
        r.s[e] = s;
        r.sc[e] = __fadd_rn(s, p.bias[e]);
    }
    tm.sync();
    for (int g = warp; g < G; g += tm.nwarp) {
        float t1 = -INFINITY, t2 = -INFINITY;
        for (int e = g * gs + lane; e < (g + 1) * gs; e += 32) {
            const float v = r.sc[e];
            if (v > t1) { t2 = t1; t1 = v; }
            else if (v > t2) { t2 = v; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float b1 = __shfl_xor_sync(0xffffffffu, t1, o), b2 = __shfl_xor_sync(0xffffffffu, t2, o);
            const float hi = fmaxf(t1, b1), lo = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
            t1 = hi;
            t2 = lo;
        }
        if (lane == 0) r.gsc[g] = __fadd_rn(t1, t2);        // gs >= 32: two members at least
    }
    tm.sync();
    // kept groups as a bit mask (every thread the same): lane g of every warp ranks group g
    uint32_t kept;
    {
        int rank = 0;
        if (lane < G) {
            const float v = r.gsc[lane];
            for (int h = 0; h < G; ++h) {
                const float u = r.gsc[h];
                rank += (u > v) || (u == v && h < lane);
            }
        }
        kept = __ballot_sync(0xffffffffu, lane < G && rank < Gk);
    }
    for (int q = tid; q < 2 * E; q += tm.nthr) {       // (expert, half) pairs on neighbouring lanes
        const int e = q >> 1, half = q & 1;
        const bool mine = kept >> (e / gs) & 1u;
        int cnt = 0;
        if (mine) {
            const float v = r.sc[e];
            for (uint32_t km = kept; km; km &= km - 1) {
                const int g = __ffs(km) - 1;
                const int b0 = g * gs + half * (gs / 2), b1 = b0 + gs / 2;
#pragma unroll 4
                for (int e2 = b0; e2 < b1; ++e2) {
                    const float u = r.sc[e2];
                    cnt += (u > v) || (u == v && e2 < e);
                }
            }
        }
        cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
        if (mine && half == 0 && cnt < k) {
            r.pick[cnt] = e;
            ps[cnt] = r.s[e];
        }
    }
    tm.sync();
    if (warp == 0) {
        const int my_e = lane < k ? r.pick[lane] : 0;
        const float my_s = lane < k ? ps[lane] : 0.f;
        double ssum = 0.0;
        for (int j = 0; j < k; ++j) ssum += (double)__shfl_sync(0xffffffffu, my_s, j);
        const float wv = lane < k ? (float)((double)my_s / ssum * (double)p.rsf) : 0.f;
        const bool keep = p.topp_thr > 0.0 ? warp_topp_keep(lane, k, wv, p.topp_thr) : true;
        const bool valid = lane < k && keep;
        const int e = valid ? my_e : -1;
        // permutation: the kept experts are distinct; position = kept experts below
        const unsigned vm = __ballot_sync(0xffffffffu, valid);
        int pos = 0;
        for (int j = 0; j < k; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e, j);
            pos += (vm >> j & 1u) && ej < e;
        }
        const int nu = __popc(vm);
        if (lane < k) {
            r.ridx[lane] = e;
            r.rw[lane] = keep ? wv : 0.f;
            r.pos[lane] = valid ? pos : -1;
            r.lead[lane] = valid;
            r.cnt[lane] = valid ? 1 : 0;
        }
        if (valid) {
            srt[pos] = lane;
            sl.e[pos] = e;
            sl.p0[pos] = pos;
            sl.nt[pos] = 1;
        }
        if (lane == 0) {
            const int nslots = nu + (p.shared ? 1 : 0);
            sl.hdr[0] = nslots;
            sl.hdr[1] = nu;
            if (p.shared) {
                sl.e[nu] = -1;
                sl.p0[nu] = 0;
                sl.nt[nu] = 1;
            }
        }
    }
    tm.sync();
    if (blockIdx.x == 0) g2_publish(p, r, sl, k, sl.hdr[1], sl.hdr[0], tm);
}

// Slot table from a permutation in memory (gate/up without fusing; down
// without a compact table): routed slots in union order, then the shared one.
// gate/up also copies `sorted` (A entries) into srt.  Ends with __syncthreads.
__device__ void g2_slots_from_perm(const G2P &p, G2Slots sl, int *srt, bool gateup)
{
    const int tid = threadIdx.x;
    if (p.tab) {
        const int nslots = p.tab[0];
        if (nslots < 0 || nslots > p.ms) {
            if (tid == 0) {
                raise_status(DERR_BADIDX);
                sl.hdr[0] = sl.hdr[1] = 0;
            }
            __syncthreads();
            return;
        }
        for (int s = tid; s < nslots; s += G2_THREADS) {
            const int4 v = *reinterpret_cast<const int4 *>(p.tab + G2_TAB_HDR + 4 * s);
            sl.e[s] = v.x;
            sl.p0[s] = v.y;
            sl.nt[s] = v.z;
        }
        if (tid == 0) {
            sl.hdr[0] = nslots;
            sl.hdr[1] = p.tab[1];
        }
        __syncthreads();
        return;
    }
    int nu = p.routed ? *p.n_union : 0;
    if (nu < 0 || nu > p.ms - 1) {
        if (tid == 0) raise_status(DERR_BADIDX);
        nu = 0;
    }
    for (int s = tid; s < nu; s += G2_THREADS) {
        int e = p.union_ids[s];
        if (e < 0 || e >= p.E) {
            raise_status(DERR_BADIDX);
            sl.e[s] = 0;
            sl.p0[s] = 0;
            sl.nt[s] = 0;
            continue;
        }
        const int o0 = p.offsets[e], o1 = p.offsets[e + 1];
        sl.e[s] = e;
        sl.p0[s] = o0;
        sl.nt[s] = o1 - o0;
    }
    if (gateup && p.routed)
        for (int i = tid; i < p.T * p.k; i += G2_THREADS) srt[i] = p.sorted[i];
    if (tid == 0) {
        sl.hdr[0] = nu + (p.shared ? 1 : 0);
        sl.hdr[1] = nu;
        if (p.shared) {
            sl.e[nu] = -1;
            sl.p0[nu] = 0;
            sl.nt[nu] = p.T;
        }
    }
    __syncthreads();
}

// This CTA's segments: its range of the slots' total cost cut into (slot,
// first warp-unit, end warp-unit) triples, seg[0] the count.  A slot's
// warp-units cost G2_BW + its tokens (at most TP) each.  Run by one warp; when
// every slot costs the same the prefix is a product, else a scan into pre.
template <int TP>
__device__ void g2_segments(const G2P &p, G2Slots sl, int nslots, int64_t *pre, int *seg)
{
    const int lane = threadIdx.x & 31;
    const int nt0 = nslots > 0 ? min(sl.nt[0], TP) : 0;
    bool same = true;
    for (int s = lane; s < nslots; s += 32) same = same && min(sl.nt[s], TP) == nt0;
    same = __all_sync(0xffffffffu, same) && nt0 > 0;
    const int64_t C = (int64_t)p.nwu * (G2_BW + nt0);          // the cost of one slot when all are the same
    int64_t Ctot;
    if (same) {
        Ctot = C * nslots;
    } else {
        int64_t run = 0;
        for (int s0 = 0; s0 < nslots; s0 += 32) {
            const int s = s0 + lane;
            int64_t cost = 0;
            if (s < nslots) {
                const int nt = sl.nt[s];
                cost = nt > 0 ? (int64_t)p.nwu * (G2_BW + min(nt, TP)) : 0;
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
        __syncwarp();
        Ctot = run;
    }
    int64_t c0, c1;
    if (Ctot < (int64_t)(0x7fffffff / gridDim.x)) {        // 32-bit arithmetic is exact
        c0 = (int)Ctot * (int)blockIdx.x / (int)gridDim.x;
        c1 = (int)Ctot * (int)(blockIdx.x + 1) / (int)gridDim.x;
    } else {
        c0 = Ctot * blockIdx.x / gridDim.x;
        c1 = Ctot * (blockIdx.x + 1) / gridDim.x;
    }
    int nseg = 0;
    for (int s0 = 0; s0 < nslots; s0 += 32) {
        const int s = s0 + lane;
        int bf = 0, be = 0;
        if (s < nslots && sl.nt[s] > 0) {
            const int cu = (int)G2_BW + min(sl.nt[s], TP);       // cost of one of the slot's warp-units
            const int64_t g0 = same ? C * s : pre[s], g1 = same ? g0 + C : pre[s + 1];
            // first unit whose cost interval starts at or after c0, and likewise for c1
            bf = c0 <= g0 ? 0 : (c0 >= g1 ? p.nwu : ((int)(c0 - g0) + cu - 1) / cu);
            be = c1 <= g0 ? 0 : (c1 >= g1 ? p.nwu : ((int)(c1 - g0) + cu - 1) / cu);
        }
        const bool has = be > bf;
        const unsigned m = __ballot_sync(0xffffffffu, has);
        if (has) {
            const int i = nseg + __popc(m & ((1u << lane) - 1u));
            seg[1 + 3 * i] = s;
            seg[2 + 3 * i] = bf;
            seg[3 + 3 * i] = be;
        }
        nseg += __popc(m);
    }
    if (lane == 0) seg[0] = nseg;
}

// ---------------------------------------------------------------- kernel

// Shared memory (offsets in G2P): slot table, srt, cost prefix, the CTA's
// segments (slot, first and end warp-unit), row maxima, route scratch, records.
template <int WB, int NDIG, int TP, int R, bool GATEUP, bool PROBE, int NJ>
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
    G2Slots sl(reinterpret_cast<int *>(sm + p.o_sl), p.ms);
    int *srt = reinterpret_cast<int *>(sm + p.o_srt);
    int64_t *pre = reinterpret_cast<int64_t *>(sm + p.o_pre);
    int *seg = reinterpret_cast<int *>(sm + p.o_seg);     // [0] count, then (slot, u0, u1) per segment
    float *rmax = reinterpret_cast<float *>(sm + p.o_rmax);
    unsigned char *recs = sm + p.o_rec;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    bool routed_now = false;
    if constexpr (GATEUP) {
        if (p.fuse && g2_route1_ok(p.T, p.E, p.G, p.k) && p.E <= G2_THREADS / 2) {
            // one token: half the CTA makes the choice from the logits while the
            // other half builds the token's record (x is an input of the call)
            if (warp < G2_NW / 2) {
                pdl_wait();            // the logits
                g2_route1(p, reinterpret_cast<int *>(sm + p.o_route), sl, srt,
                          G2Team{tid, G2_THREADS / 2, warp, G2_NW / 2, 1});
            } else {
                g2_build<WB, NDIG, true>(p, recs, p.T, [](int i, int64_t &row) { row = i; return true; }, true, rmax,
                                         G2Team{tid - G2_THREADS / 2, G2_THREADS / 2, warp - G2_NW / 2, G2_NW / 2, 2});
            }
            __syncthreads();
            pdl_trigger();
            routed_now = true;
        } else {
            // the records of every token, before the dependency wait: x is an input
            // of the call, so this overlaps the kernels before
            g2_build<WB, NDIG, true>(p, recs, p.T, [](int i, int64_t &row) { row = i; return true; }, true, rmax);
        }
    }
    if (!routed_now) {
        pdl_wait();            // gate/up: the logits or the permutation; down: h, from the kernels before
        pdl_trigger();
        if (GATEUP && p.fuse) {
            if (g2_route1_ok(p.T, p.E, p.G, p.k)) g2_route1(p, reinterpret_cast<int *>(sm + p.o_route), sl, srt);
            else g2_route(p, reinterpret_cast<int *>(sm + p.o_route), sl, srt);
        } else {
            g2_slots_from_perm(p, sl, srt, GATEUP);
        }
    }
    const int nslots = sl.hdr[0], nu = sl.hdr[1];
    uint32_t *hmx = reinterpret_cast<uint32_t *>(sm + p.o_hmx);
    if (warp == 0) {
        g2_segments<TP>(p, sl, nslots, pre, seg);
        if (GATEUP && p.hmax) {
            __syncwarp();
            for (int i = lane; i < seg[0] * TP; i += 32) hmx[i] = 0u;
        }
    }
    __syncthreads();
    const int nseg = seg[0];
    QRX_CHECK_ONLY(const int64_t n_pos = p.routed ? (int64_t)p.T * p.k : 0;)
    QRX_CHECK_ONLY(const int64_t n_out = max(n_pos, p.shared ? p.sh_out_row0 + p.T : (int64_t)0);)

    // NJ > 0: rows of 32 * NJ chunks, fixed at compile time (LPR = 32)
    const int LPR = NJ > 0 ? 32 : p.lpr, nj = NJ > 0 ? NJ : p.nj;
    const int cl = lane % LPR, grp = lane / LPR;
    const G2Rec RL = g2_rec(NDIG, p.K, p.cpr);
    // after the butterfly (V <= LPR) lane cl holds value cl / rep: that value's
    // row (and for gate/up: gate, with the up value on lane cl + rep)
    const int rep = V <= LPR ? LPR / V : 1;
    const int my_idx = cl / rep;
    const int my_i = (my_idx / NM) % R;
    const bool writer = V <= LPR && cl % rep == 0 && (!GATEUP || (my_idx & 1) == 0);

    const int plen = GATEUP ? nseg : p.slot_cap;          // segments per phase
    for (int ph0 = 0; ph0 < nseg; ph0 += plen) {
        const int ph1 = min(nseg, ph0 + plen);
        if constexpr (!GATEUP) {
            if (ph0 > 0) __syncthreads();                 // every warp is done with the last phase's records
            g2_build<WB, NDIG, false>(p, recs, (ph1 - ph0) * TP,
                               [&](int i, int64_t &row) {
                                   const int s = seg[1 + 3 * (ph0 + i / TP)], t = i % TP;
                                   if (t >= min(sl.nt[s], TP)) return false;
                                   row = s < nu ? (int64_t)sl.p0[s] + t : p.sh_in_row0 + t;
                                   return true;
                               },
                               false, rmax);
        }
        int rec[TP];           // shared-memory offsets of the slot's token records
        int64_t orow[TP];
        int corr[TP][NP];      // NDIG = 3: OFF * (this lane's digit sums over its chunks), per plane
        float sig[TP];
#pragma unroll
        for (int t = 0; t < TP; ++t) {
            rec[t] = p.o_rec;
            orow[t] = 0;
            sig[t] = 1.f;
#pragma unroll
            for (int pl = 0; pl < NP; ++pl) corr[t][pl] = 0;
        }
        int ntot = 0;
        for (int j = ph0; j < ph1; ++j) ntot += seg[3 + 3 * j] - seg[2 + 3 * j];
        const int f0 = (int)((int64_t)ntot * warp / G2_NW), f1 = (int)((int64_t)ntot * (warp + 1) / G2_NW);
        int j = ph0, jbase = 0, cur_s = -1, nt = 0, e = 0;
        bool routed = false;
        bool have0 = false;            // chunk 0 of this warp-unit was loaded by the one before
        uint4 bufA[NM][R], bufB[NM][R];
        for (int f = f0; f < f1; ++f) {
            while (f >= jbase + seg[3 + 3 * j] - seg[2 + 3 * j]) {
                jbase += seg[3 + 3 * j] - seg[2 + 3 * j];
                ++j;
            }
            const int s = seg[1 + 3 * j], u = seg[2 + 3 * j] + (f - jbase);
            if (s != cur_s) {
                // ---- enter a slot: its tokens, their records, this lane's corrections
                routed = s < nu;
                e = routed ? sl.e[s] : 0;
                const int p0 = routed ? sl.p0[s] : 0;
                nt = min(sl.nt[s], TP);
                bool ok = true;
#pragma unroll
                for (int i = 0; i < TP; ++i) {
                    const int ii = min(i, max(nt - 1, 0));
                    if (routed) {
                        QRX_CHECK_OR((int64_t)p0 + ii < n_pos, ok = false);
                        orow[i] = p0 + ii;
                        if constexpr (GATEUP) {
                            const int a = srt[p0 + ii];
                            QRX_CHECK_OR(a >= 0 && a / p.k < p.T, ok = false);
                            rec[i] = p.o_rec + (a / p.k) * p.rec_bytes;
                        } else {
                            rec[i] = p.o_rec + ((j - ph0) * TP + ii) * p.rec_bytes;
                        }
                    } else {
                        orow[i] = p.sh_out_row0 + ii;
                        rec[i] = GATEUP ? p.o_rec + ii * p.rec_bytes : p.o_rec + ((j - ph0) * TP + ii) * p.rec_bytes;
                    }
                }
                if (!ok) return;
                if constexpr (NDIG == 3) {
#pragma unroll
                    for (int t = 0; t < TP; ++t) {
                        sig[t] = *reinterpret_cast<const float *>(sm + rec[t] + RL.hdr);
                        int s0 = 0, s1 = 0, s2 = 0;
                        for (int jj = 0; jj < nj; ++jj) {
                            const int4 c4 = *reinterpret_cast<const int4 *>(sm + rec[t] + RL.csum + (cl + LPR * jj) * 16);
                            s0 += c4.x;
                            s1 += c4.y;
                            s2 += c4.z;
                        }
                        corr[t][0] = F::OFF * s0;
                        corr[t][1] = F::OFF * s1;
                        corr[t][2] = F::OFF * s2;
                    }
                }
                cur_s = s;
            }
            // ---- one warp-unit: this lane's rows, their row pointers and (writers) scales
            const int r0 = u * p.rw;
            const uint8_t *wrow[NM][R];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const uint8_t *base = routed ? p.m[m].q + (int64_t)e * p.m[m].sq : p.msh[m].q;
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    const int row = min(r0 + grp + p.gpw * i, p.rows - 1);     // a row past the end is read, unused
                    wrow[m][i] = base + (int64_t)row * p.row_bytes;
                }
            }
            float sc0 = 0.f, sc1 = 0.f;
            const int wr_row = r0 + grp + p.gpw * my_i;
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
            auto load = [&](int jc, uint4 (&b)[NM][R]) {
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int i = 0; i < R; ++i) b[m][i] = ld_stream16(wrow[m][i] + (size_t)(cl + LPR * jc) * 16);
            };
            // chunk jc of every row of this lane, against every token of the slot
            auto compute = [&](int jc, const uint4 (&b)[NM][R]) {
                const int c = cl + LPR * jc;
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
                                        const int64_t row = r0 + grp + p.gpw * i;
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
            // chunk 0 of the warp's next unit (its rows found from the segment list)
            const bool has_next = f + 1 < f1;
            auto load_next = [&](uint4 (&b)[NM][R]) {
                int j2 = j, jb2 = jbase;
                while (f + 1 >= jb2 + seg[3 + 3 * j2] - seg[2 + 3 * j2]) {
                    jb2 += seg[3 + 3 * j2] - seg[2 + 3 * j2];
                    ++j2;
                }
                const int s2 = seg[1 + 3 * j2], u2 = seg[2 + 3 * j2] + (f + 1 - jb2);
                const bool rt2 = s2 < nu;
                const int e2 = rt2 ? sl.e[s2] : 0;
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const uint8_t *base = rt2 ? p.m[m].q + (int64_t)e2 * p.m[m].sq : p.msh[m].q;
#pragma unroll
                    for (int i = 0; i < R; ++i) {
                        const int row = min(u2 * p.rw + grp + p.gpw * i, p.rows - 1);
                        b[m][i] = ld_stream16(base + (int64_t)row * p.row_bytes + (size_t)cl * 16);
                    }
                }
            };
            // the streaming loop: chunk jc + 1's loads are issued before chunk jc
            // is computed, and the next unit's chunk 0 before this unit's last
            if (!have0) load(0, bufA);
#pragma unroll 1
            for (int jc = 0; jc < nj; jc += 2) {
                if (jc + 1 < nj) load(jc + 1, bufB);
                else if (has_next) load_next(bufB);
                compute(jc, bufA);
                if (jc + 2 < nj) load(jc + 2, bufA);
                else if (jc + 1 < nj && has_next) load_next(bufA);
                if (jc + 1 < nj) compute(jc + 1, bufB);
            }
            have0 = has_next;
            if (has_next && (nj & 1)) {      // an odd chunk count left the next unit's chunk 0 in bufB
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int i = 0; i < R; ++i) bufA[m][i] = bufB[m][i];
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
                        } else {
                            x = facc[t][m][i];
                        }
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
                const int row = r0 + grp + p.gpw * i;
                if (t >= nt || row >= p.rows) return;
                const int64_t o = g2_pick(orow, t);
                QRX_CHECK_OR(o >= 0 && o < n_out, return);
                const float sg = NDIG == 3 ? g2_pick(sig, t) : 1.f;
                if constexpr (GATEUP) {
                    const float hv = silu_mul(s0 * (sg * tot), s1 * (sg * upv));
                    p.out[o * p.out_ld + row] = hv;
                    if (p.hmax) atomicMax(hmx + j * TP + t, __float_as_uint(fabsf(hv)));
                } else
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
                    const int row = min(r0 + grp + p.gpw * i, p.rows - 1);
                    const float s0 = routed ? p.m[0].s[(int64_t)e * p.m[0].ss + row] : p.msh[0].s[row];
                    const float s1 = GATEUP ? (routed ? p.m[NM - 1].s[(int64_t)e * p.m[NM - 1].ss + row] : p.msh[NM - 1].s[row]) : 0.f;
                    emit(idx, v[q], GATEUP ? v[q + NM - 1] : 0.f, s0, s1);
                }
            }
        }
    }
    if constexpr (GATEUP) {
        if (p.hmax) {
            // the CTA's row maxima of h, one global raise per (segment, token)
            __syncthreads();
            for (int q = tid; q < nseg * TP; q += G2_THREADS) {
                const int s = seg[1 + 3 * (q / TP)], t = q % TP;
                if (t >= min(sl.nt[s], TP) || hmx[q] == 0u) continue;
                const int64_t o = s < nu ? (int64_t)sl.p0[s] + t : p.sh_out_row0 + t;
                atomicMax(p.hmax + o, hmx[q]);
            }
        }
    }
    if constexpr (!GATEUP) {
        if (p.comb) {
            // weighted combine: one arrival per (slot, row group) of this CTA's
            // range; the arrival that completes a row group (every slot written)
            // adds its rows, for every token, in ascending j onto the shared rows
            int *lst = reinterpret_cast<int *>(sm + p.o_route);       // the groups this CTA completes
            auto comb_rows = [&](int u, int q0, int dq) {            // row group u, items q0, q0 + dq, ...
                for (int q = q0; q < p.T * p.rw; q += dq) {
                    const int t = q / p.rw, row = u * p.rw + q % p.rw;
                    if (row >= p.rows) continue;
                    float acc = p.shared ? __ldcg(p.out + (p.sh_out_row0 + t) * p.out_ld + row) : 0.f;
                    for (int jk = 0; jk < p.k; ++jk) {
                        const int64_t a = (int64_t)t * p.k + jk;
                        const float wj = p.cw[a];
                        const int pos = p.cinv[a];
                        if (pos < 0) continue;
                        QRX_CHECK_OR(pos < (int64_t)p.T * p.k, continue);
                        acc = fmaf(wj, __ldcg(p.out + (int64_t)pos * p.out_ld + row), acc);
                    }
                    p.cout[(int64_t)t * p.rows + row] = acc;
                }
            };
            __threadfence();
            __syncthreads();
            if (tid == 0) lst[0] = 0;
            __syncthreads();
            int nall = 0;
            for (int jj = 0; jj < nseg; ++jj) nall += seg[3 + 3 * jj] - seg[2 + 3 * jj];
            for (int q = tid; q < nall; q += G2_THREADS) {
                int jj = 0, qb = 0;
                while (q >= qb + seg[3 + 3 * jj] - seg[2 + 3 * jj]) {
                    qb += seg[3 + 3 * jj] - seg[2 + 3 * jj];
                    ++jj;
                }
                const int u = seg[2 + 3 * jj] + (q - qb);
                if (atomicAdd(p.cnt + u, 1) == nslots - 1) {
                    __threadfence();
                    const int li = atomicAdd(lst, 1);
                    if (li < G2_CLIST) lst[1 + li] = u;
                    else comb_rows(u, 0, 1);                          // list full: this thread does it
                }
            }
            __syncthreads();
            const int nl = min(lst[0], G2_CLIST), per = p.T * p.rw;
            for (int q = tid; q < nl * per; q += G2_THREADS) comb_rows(lst[1 + q / per], q % per, per);
        }
    }
}

// ---------------------------------------------------------------- host side
struct G2Plan {
    G2P p;
    int tp, r;
};

// Geometry for one projection: `nm` matrices of `rows` rows x K codes at wbits,
// activations with ndig digit planes, calls of T <= G2_TMAX tokens over E
// experts at top-k (route: the fused selection's groups G, kept Gk; G = 0: no
// fused selection).  R (rows per lane per matrix) is 2 for gate/up and 4 for
// down: four row chunks per lane per step, double-buffered (halved for several
// tokens with f32 / bf16 digits, or int2, to fit the accumulators in
// registers).  gate/up holds every token's record; down holds the records of
// slot_cap slots at a time.
static inline bool g2_plan(G2Plan &pl, int wbits, int ndig, int K, int rows, int nm, int T, int E, int k, int G = 0,
                           int Gk = 0)
{
    G2P &p = pl.p;
    p = G2P{};
    if (T < 1 || T > G2_TMAX || rows < 1 || E < 1 || k < 1 || k > 32) return false;
    pl.tp = T == 1 ? 1 : (T == 2 ? 2 : 4);
    pl.r = nm == 2 ? 2 : 4;
    if (pl.tp >= 2 && (ndig == 3 || wbits == 2)) pl.r /= 2;   // several tokens' sums, or int2's wide unpack
    p.K = K;
    p.rows = rows;
    p.row_bytes = K * wbits / 8;
    if (K % 32 || p.row_bytes % 16) return false;
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
    p.nwu = (rows + p.rw - 1) / p.rw;
    p.rec_bytes = (g2_rec(ndig, K, p.cpr).bytes + 127) & ~127;
    const int A = T * k;
    p.ms = (E < A ? E : A) + 1;
    auto al = [](int v, int a) { return (v + a - 1) / a * a; };
    int o = 0;
    p.o_sl = o;
    o = al(o + (4 + 3 * p.ms) * 4, 16);
    p.o_srt = o;
    o = al(o + A * 4, 16);
    p.o_pre = o;
    o = al(o + (p.ms + 1) * 8, 16);
    p.o_seg = o;
    o = al(o + (1 + 3 * p.ms) * 4, 16);
    p.o_hmx = o;                                   // gate/up: largest |h| per (segment, token)
    o = al(o + p.ms * pl.tp * 4, 16);
    p.o_route = o;
    if (G > 0) o = al(o + G2RouteSm::ints(T, E, G, Gk, k) * 4, 16);
    else if (nm == 1) o = al(o + (1 + G2_CLIST) * 4, 16);         // down: the combine's list
    p.o_rmax = o;
    if (nm == 2) {
        p.nrec = T;
        p.slot_cap = p.ms;
        o = al(o + T * G2_NW * 4, 128);
    } else {
        const int per = pl.tp * (p.rec_bytes + G2_NW * 4);
        int cap = (G2_SMEM_MAX - 128 - o) / per;
        if (cap > p.ms) cap = p.ms;
        if (cap < 1) return false;
        p.slot_cap = cap;
        p.nrec = cap * pl.tp;
        o = al(o + p.nrec * G2_NW * 4, 128);
    }
    p.o_rec = o;
    o += p.nrec * p.rec_bytes;
    p.smem = o;
    return o <= G2_SMEM_MAX;
}

template <int WB, int ND, int TP, int R, bool GU, bool PR, int NJ = 0>
static cudaError_t g2_go(const G2P &p, int grid, cudaStream_t st)
{
    auto kern = k_gemv2<WB, ND, TP, R, GU, PR, NJ>;
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
    // rows of the common shapes (hidden 6144, expert intermediate 2048) with the chunk count fixed
    if constexpr (!PR) {
        if (pl.p.lpr == 32 && wbits == 4 && ndig == 3 && pl.tp == 1 && pl.r == R1) {
            if (pl.p.nj == 6) return g2_go<4, 3, 1, R1, GU, PR, 6>(pl.p, grid, st);
            if (pl.p.nj == 2) return g2_go<4, 3, 1, R1, GU, PR, 2>(pl.p, grid, st);
        }
    }
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
    p.offsets = const_cast<int32_t *>(a.offsets);
    p.sorted = const_cast<int32_t *>(a.sorted);
    p.union_ids = const_cast<int32_t *>(a.union_ids);
    p.n_union = const_cast<int32_t *>(a.n_union);
    p.E = a.E;
    p.k = a.k;
    p.T = a.T;
    p.afmt = a.afmt;
}

static inline G2Mat g2_mat(const MatRef &m) { return G2Mat{m.q, m.s, m.sq, m.ss}; }

static inline int g2_ndig(const FfnArgs &a) { return a.afmt == QRX_A_Q8_0 ? 1 : 3; }

bool g2_use(const FfnArgs &a)
{
    if (a.T < 1 || a.T > G2_TMAX) return false;
    G2Plan pg, pd;
    return g2_plan(pg, a.wbits, g2_ndig(a), a.H, a.I, 2, a.T, a.E, a.k) &&
           g2_plan(pd, a.wbits, g2_ndig(a), a.I, a.H, 1, a.T, a.E, a.k);
}

bool g2_fuse_ok(const FfnArgs &a, int G, int Gk)
{
    if (!g2_use(a) || G < 1 || a.E % G) return false;
    G2Plan pg;
    return g2_plan(pg, a.wbits, g2_ndig(a), a.H, a.I, 2, a.T, a.E, a.k, G, Gk);
}

// Entries of the combine counter array for the down projection of this call.
int g2_down_groups(const FfnArgs &a)
{
    G2Plan pd;
    return g2_plan(pd, a.wbits, g2_ndig(a), a.I, a.H, 1, a.T, a.E, a.k) ? pd.p.nwu : 0;
}

static void g2_gateup_args(G2P &p, const FfnArgs &a, int32_t *probe)
{
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
}

static void g2_down_args(G2P &p, const FfnArgs &a, int32_t *probe)
{
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
}

cudaError_t launch_g2_gateup(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = g2_ndig(a);
    G2Plan pl;
    if (!g2_plan(pl, a.wbits, ndig, a.H, a.I, 2, a.T, a.E, a.k)) return cudaErrorInvalidValue;
    g2_gateup_args(pl.p, a, probe);
    if (probe) return ndig == 1 ? g2_dispatch<true, true>(pl, a.wbits, ndig, num_sms, st) : cudaErrorInvalidValue;
    return g2_dispatch<true, false>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_g2_down(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = g2_ndig(a);
    G2Plan pl;
    if (!g2_plan(pl, a.wbits, ndig, a.I, a.H, 1, a.T, a.E, a.k)) return cudaErrorInvalidValue;
    g2_down_args(pl.p, a, probe);
    if (probe) return ndig == 1 ? g2_dispatch<false, true>(pl, a.wbits, ndig, num_sms, st) : cudaErrorInvalidValue;
    return g2_dispatch<false, false>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_g2_gateup_fused(const FfnArgs &a, const G2Fuse &f, int num_sms, cudaStream_t st)
{
    const int ndig = g2_ndig(a);
    G2Plan pl;
    if (!a.routed || !g2_plan(pl, a.wbits, ndig, a.H, a.I, 2, a.T, a.E, a.k, f.G, f.Gk)) return cudaErrorInvalidValue;
    G2P &p = pl.p;
    g2_gateup_args(p, a, nullptr);
    p.fuse = 1;
    p.logits = f.logits;
    p.bias = f.bias;
    p.G = f.G;
    p.Gk = f.Gk;
    p.rsf = f.rsf;
    p.topp_thr = f.topp_thr;
    p.idx = f.idx;
    p.w = f.w;
    p.usage = f.usage;
    p.counts = f.counts;
    p.inv = f.inv;
    p.tab_out = f.tab;
    p.hmax = f.hmax;
    p.cnt = f.cnt;
    p.ncnt = f.cnt ? g2_down_groups(a) : 0;
    return g2_dispatch<true, false>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_g2_down_fused(const FfnArgs &a, const G2Fuse &f, int num_sms, cudaStream_t st)
{
    const int ndig = g2_ndig(a);
    G2Plan pl;
    if (!a.routed || !g2_plan(pl, a.wbits, ndig, a.I, a.H, 1, a.T, a.E, a.k)) return cudaErrorInvalidValue;
    G2P &p = pl.p;
    g2_down_args(p, a, nullptr);
    p.tab = f.tab;
    p.hmax = f.hmax;
    if (f.out) {
        p.comb = 1;
        p.cnt = f.cnt;
        p.ncnt = p.nwu;
        p.cw = f.w;
        p.cinv = f.inv;
        p.cout = f.out;
    }
    return g2_dispatch<false, false>(pl, a.wbits, ndig, num_sms, st);
}

}  // namespace qrx
