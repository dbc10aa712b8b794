// k_gmma.cuh -- multi-token expert FFN (calls of 2 to 64 tokens): the batch
// union streamed from HBM like the decode GEMV (k_gemv2.cuh), with the dot
// products of a weight row against all of its slot's tokens on the tensor
// cores (mma.sync m16n8k32, unsigned 8-bit weights x signed 8-bit digits ->
// exact int32).
//
// README "JustVugg/colibri", section "已实现的功能": batch-union MoE (each
// unique expert read once for all positions routed to it), packed int4 / int8
// weights with per-row scales dequantised on use, Q8_0-style int8-activation
// integer dots; the expert is a SwiGLU FFN, h = silu(s_g Q_g x) * (s_u Q_u x),
// y = s_d Q_d h.
//
// Work.  Slots (experts of the union, then the shared expert) with more
// tokens than one pass takes (NTOK) are split into instances of at most NTOK
// tokens, each streaming the expert's rows once.  A warp-unit is (instance,
// 16 consecutive rows of each matrix); units are cut into cost ranges per CTA
// and contiguous runs per warp as in the decode GEMV.  A CTA works through its
// instances in phases: the records of a phase's tokens (the activation digit
// planes, built by the whole CTA) are held in shared memory.
//
// A warp streams its 16 rows (of gate and up, or of down) 64 bytes per row at
// a time: lane (g, t) (g = lane / 4, t = lane % 4) loads bytes 16 t .. 16 t + 15
// of rows g and g + 8 (128-bit loads that skip L1, one step ahead), stores
// them to a 16-row tile of its own in shared memory, and ldmatrix hands every
// lane word t of each 16-byte piece of rows g and g + 8 -- the A fragment of
// m16n8k32 up to the order of k inside a block, which the activation records
// share: for int4 the low nibbles of word t (codes 8t, 8t+2, 8t+4, 8t+6) fill
// k = 4t .. 4t+3 and the high nibbles (codes 8t+1, ...) k = 16+4t .. 16+4t+3,
// which are the record's digit words 2t and 2t+1 of that block (the B
// fragment of column n on lanes with g = n); for int8 word t of pieces 2m and
// 2m+1 are codes 4t .. 4t+3 and 16+4t .. 16+4t+3 of block m.  Columns are
// (token, digit plane) pairs: token * 3 + plane for f32 / bf16 activations
// (three planes of the 22-bit fixed point, each column's int32 sum exact over
// all of K), the token for Q8_0 (one 32-code block per mma, started from the
// block's offset correction and scaled by the token's d_b in f32).  int4
// codes enter as offset binary (code + 8); the offset is removed through the
// digit sums (per block for Q8_0, per row and plane for the fixed point).
// The down projection with the fixed point skips the tile: each lane's own
// 16 bytes of rows g and g + 8 (block 4 s + t of step s for int4, half a block
// for int8) are its A fragments -- word j's low and high nibbles (int4), or
// words 2 j and 2 j + 1 (int8), fill k = 4 t .. 4 t + 3 and 16 + 4 t .. of mma
// j -- and the B fragments are the matching digit words of record chunk
// 4 s + t; the sums are exact over all of K, so the k order is free.
#pragma once
#include "k_gemv2.cuh"

namespace qrx {

constexpr int GM_ROWS = 16;                       // rows of each matrix per warp-unit
constexpr int GM_SCB = 64;                        // bytes of a row per streaming step
constexpr int GM_TSTRIDE = 80;                    // bytes per row of a warp's tile (64 + 16: ldmatrix without bank conflicts)
constexpr int GM_COST_ROWS = 16;                  // cost of a warp-unit: 16 for its bytes, plus one per token
constexpr int GM_STAGES = 3;                      // tiles in a warp's copy ring

__device__ __forceinline__ void gm_cp16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void gm_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void gm_wait_groups() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void gm_mma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1, bool uns)
{
    if (uns)
        asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void gm_ldsm4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Split every slot of more than ntok tokens into instances of at most ntok
// tokens (same expert, consecutive positions), in place in the slot table
// (capacity p.ms).  Run by one warp after the slot table is complete; the
// split keeps the slots' order, routed ones first.
__device__ void gm_split(const G2P &p, G2Slots sl, int ntok)
{
    const int lane = threadIdx.x & 31;
    const int nslots = sl.hdr[0], nu = sl.hdr[1];
    // instances per slot, their prefix (one pass of lanes over the slots)
    int total = 0, nu2 = 0;
    for (int s = 0; s < nslots; ++s) {
        const int n = max(1, (sl.nt[s] + ntok - 1) / ntok);
        total += n;
        if (s < nu) nu2 += n;
    }
    if (total > p.ms) {                            // cannot happen: the plan sizes the table for it
        if (lane == 0) raise_status(DERR_BOUNDS);
        total = nslots;
        nu2 = nu;
        ntok = 1 << 30;
    }
    __syncwarp();
    // fill from the back so that no entry is overwritten before it is read
    if (lane == 0) {
        int d = total;
        for (int s = nslots - 1; s >= 0; --s) {
            const int e = sl.e[s], p0 = sl.p0[s], nt = sl.nt[s];
            const int n = max(1, (nt + ntok - 1) / ntok);
            for (int i = n - 1; i >= 0; --i) {
                --d;
                sl.e[d] = e;
                sl.p0[d] = p0 + i * ntok;
                sl.nt[d] = min(ntok, nt - i * ntok);
            }
        }
        sl.hdr[0] = total;
        sl.hdr[1] = nu2;
    }
    __syncwarp();
}

// This CTA's segments of the instances' total cost (cost of a warp-unit:
// GM_COST_ROWS + its tokens).  Run by one warp; pre: nslots + 1 int64.
__device__ void gm_segments(const G2P &p, G2Slots sl, int nslots, int64_t *pre, int *seg)
{
    const int lane = threadIdx.x & 31;
    int64_t run = 0;
    for (int s0 = 0; s0 < nslots; s0 += 32) {
        const int s = s0 + lane;
        int64_t cost = 0;
        if (s < nslots && sl.nt[s] > 0) cost = (int64_t)p.nwu * (GM_COST_ROWS + sl.nt[s]);
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
    const int64_t Ctot = run;
    const int64_t c0 = Ctot * blockIdx.x / gridDim.x, c1 = Ctot * (blockIdx.x + 1) / gridDim.x;
    int nseg = 0;
    for (int s0 = 0; s0 < nslots; s0 += 32) {
        const int s = s0 + lane;
        int bf = 0, be = 0;
        if (s < nslots && sl.nt[s] > 0) {
            const int64_t cu = GM_COST_ROWS + sl.nt[s], g0 = pre[s], g1 = pre[s + 1];
            bf = c0 <= g0 ? 0 : (c0 >= g1 ? p.nwu : (int)((c0 - g0 + cu - 1) / cu));
            be = c1 <= g0 ? 0 : (c1 >= g1 ? p.nwu : (int)((c1 - g0 + cu - 1) / cu));
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
// Shared memory (offsets in G2P): slot table, srt, cost prefix, segments, row
// maxima, plane digit totals (o_route: per record 4 ints), warp tiles (o_hmx:
// G2_NW tiles of tile bytes), records.
template <int WB, int NDIG, int NTL, bool GATEUP>
__global__ void __launch_bounds__(G2_THREADS, 1) k_gmma(const __grid_constant__ G2P p)
{
    using F = Fmt<WB>;
    constexpr int NM = GATEUP ? 2 : 1;
    constexpr int NC = 8 * NTL;                          // columns per pass
    constexpr int NTOK = NDIG == 3 ? NC / 3 : NC;        // tokens per pass
    constexpr int NQ = F::DW / 4;
    constexpr int NBLK = WB == 4 ? 4 : (WB == 2 ? 8 : 2);  // mmas per matrix and 64-byte step
    // down projection with the fixed point (three planes, exact sums over all of
    // K): the A fragments come straight from the lane's loads, in a k order the
    // records match.  Q8_0 needs one block per mma, which the tile and ldmatrix
    // arrange; gate/up keeps the tile ring too, which measured faster there
    // (two matrices: twice the loads per step in flight behind the copies)
    constexpr bool RD = NDIG == 3 && !GATEUP;
    static_assert(WB == 4 || WB == 8 || (WB == 2 && NDIG == 3), "int4 or int8 weights, or int2 with the fixed point");
    extern __shared__ __align__(128) unsigned char sm[];
    G2Slots sl(reinterpret_cast<int *>(sm + p.o_sl), p.ms);
    int *srt = reinterpret_cast<int *>(sm + p.o_srt);
    int64_t *pre = reinterpret_cast<int64_t *>(sm + p.o_pre);
    int *seg = reinterpret_cast<int *>(sm + p.o_seg);
    float *rmax = reinterpret_cast<float *>(sm + p.o_rmax);
    int *tot = reinterpret_cast<int *>(sm + p.o_route);  // [record][4]: OFF * digit total per plane
    unsigned char *recs = sm + p.o_rec;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    unsigned char *tile = sm + p.o_hmx + warp * p.ntile;
    const uint32_t tile_s = (uint32_t)__cvta_generic_to_shared(tile);
    const G2Rec RL = g2_rec(NDIG, p.K, p.cpr);

    // OFF times each record's digit total per plane (fixed point, int4), records [i0, i1)
    auto totals = [&](int i0, int i1) {
        if constexpr (NDIG == 3 && WB != 8) {
            for (int q = warp; q < (i1 - i0) * 3; q += G2_NW) {
                const int i = i0 + q / 3, pl = q % 3;
                const unsigned char *rec = recs + (size_t)i * p.rec_bytes;
                int sacc = 0;
                for (int c = lane; c < p.cpr; c += 32) sacc += reinterpret_cast<const int *>(rec + RL.csum + (size_t)c * 16)[pl];
#pragma unroll
                for (int o = 16; o; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
                if (lane == 0) tot[i * 4 + pl] = F::OFF * sacc;
            }
            __syncthreads();
        }
    };
    const bool allrec = GATEUP && p.allrec;
    if (allrec) {
        // every token's record, before the dependency wait: x is an input of the call
        g2_build<WB, NDIG, false>(p, recs, p.T, [](int i, int64_t &row) { row = i; return true; }, true, rmax);
        totals(0, p.T);
    }
    pdl_wait();            // the permutation and (down) h, from the kernels before
    pdl_trigger();
    g2_slots_from_perm(p, sl, srt, GATEUP);
    if (warp == 0) {
        gm_split(p, sl, NTOK);
        gm_segments(p, sl, sl.hdr[0], pre, seg);
    }
    __syncthreads();
    const int nu = sl.hdr[1], nseg = seg[0];
    QRX_CHECK_ONLY(const int64_t n_pos = p.routed ? (int64_t)p.T * p.k : 0;)
    QRX_CHECK_ONLY(const int64_t n_out = max(n_pos, p.shared ? p.sh_out_row0 + p.T : (int64_t)0);)

    const int plen = allrec ? nseg : p.slot_cap;
    for (int ph0 = 0; ph0 < nseg; ph0 += plen) {
        const int ph1 = min(nseg, ph0 + plen);
        if (ph0 > 0) __syncthreads();                     // every warp is done with the last phase's records
        // records of the phase's tokens: instance j's token i at record (j - ph0) * NTOK + i
        bool ok = true;
        if (!allrec) g2_build<WB, NDIG, false>(p, recs, (ph1 - ph0) * NTOK,
                                  [&](int i, int64_t &row) {
                                      const int s = seg[1 + 3 * (ph0 + i / NTOK)], tk = i % NTOK;
                                      if (tk >= sl.nt[s]) return false;
                                      const int q = sl.p0[s] + tk;
                                      if (s < nu) {
                                          if constexpr (GATEUP) {
                                              const int a = srt[q];
                                              QRX_CHECK_OR(a >= 0 && a / p.k < p.T, { ok = false; return false; });
                                              row = a / p.k;
                                          } else {
                                              row = q;
                                          }
                                      } else {
                                          row = GATEUP ? q : p.sh_in_row0 + q;
                                      }
                                      return true;
                                  },
                                  GATEUP, rmax);
        if (!ok) return;
        if (!allrec) totals(0, (ph1 - ph0) * NTOK);
        int ntot = 0;
        for (int j = ph0; j < ph1; ++j) ntot += seg[3 + 3 * j] - seg[2 + 3 * j];
        const int f0 = (int)((int64_t)ntot * warp / G2_NW), f1 = (int)((int64_t)ntot * (warp + 1) / G2_NW);
        int j = ph0, jbase = 0;
        for (int f = f0; f < f1; ++f) {
            while (f >= jbase + seg[3 + 3 * j] - seg[2 + 3 * j]) {
                jbase += seg[3 + 3 * j] - seg[2 + 3 * j];
                ++j;
            }
            const int s = seg[1 + 3 * j], u = seg[2 + 3 * j] + (f - jbase);
            const bool routed = s < nu;
            const int e = routed ? sl.e[s] : 0;
            const int p0 = sl.p0[s], nt = min(sl.nt[s], NTOK);
            const int rbase = (j - ph0) * NTOK;              // the instance's first record
            // record of the instance's token tk: the token's own (allrec) or the phase's
            auto recidx = [&](int tk) -> int {
                if (!allrec) return rbase + tk;
                return routed ? srt[p0 + tk] / p.k : p0 + tk;
            };
            const int r0 = u * GM_ROWS;
            // this lane's two rows of each matrix, 16 bytes at 16 t of every 64-byte step
            const uint8_t *wa[NM], *wb[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const uint8_t *base = routed ? p.m[m].q + (int64_t)e * p.m[m].sq : p.msh[m].q;
                wa[m] = base + (int64_t)min(r0 + g, p.rows - 1) * p.row_bytes + 16 * t;
                wb[m] = base + (int64_t)min(r0 + g + 8, p.rows - 1) * p.row_bytes + 16 * t;
            }
            // B operand: column 8 jj + g of n-tile jj -> (token, plane)
            int boff[NTL];          // record offset of the column's plane (-1: no such token)
#pragma unroll
            for (int jj = 0; jj < NTL; ++jj) {
                const int col = 8 * jj + g;
                const int tk = NDIG == 3 ? col / 3 : col, pl = NDIG == 3 ? col % 3 : 0;
                boff[jj] = tk < nt ? p.o_rec + recidx(tk) * p.rec_bytes + pl * NQ * p.cpr * 16 : -1;
            }
            // Q8_0: the tokens of this lane's accumulator columns 8 jj + 2 t, + 1
            int coff[NTL][2];
#pragma unroll
            for (int jj = 0; jj < NTL; ++jj)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int tk = 8 * jj + 2 * t + h;
                    coff[jj][h] = NDIG == 1 && tk < nt ? p.o_rec + recidx(tk) * p.rec_bytes + RL.hdr : -1;
                }
            int acc[NM][NTL][4];
            float facc[NM][NTL][4];
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int jj = 0; jj < NTL; ++jj)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[m][jj][q] = 0;
                        facc[m][jj][q] = 0.f;
                    }
            const int nsc = p.row_bytes / GM_SCB;
            constexpr int TB = NM * GM_ROWS * GM_TSTRIDE;      // bytes of one tile
            // the copies of step sc into tile sc % GM_STAGES (16 bytes per lane per row)
            auto issue = [&](int sc) {
                if (sc < nsc) {
                    const uint32_t tb = tile_s + (sc % GM_STAGES) * TB;
#pragma unroll
                    for (int m = 0; m < NM; ++m) {
                        gm_cp16(tb + (m * 16 + g) * GM_TSTRIDE + 16 * t, wa[m] + (size_t)sc * GM_SCB);
                        gm_cp16(tb + (m * 16 + g + 8) * GM_TSTRIDE + 16 * t, wb[m] + (size_t)sc * GM_SCB);
                    }
                }
                gm_commit();                                   // one group per step, empty past the end
            };
            auto step = [&](int sc) {
                const uint32_t tb = tile_s + (sc % GM_STAGES) * TB;
                // aw[m][piece][half]: word t of 16-byte piece `piece` of row g (half 0) or g + 8 (half 1)
                uint32_t aw[NM][4][2];
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int xq = 0; xq < 2; ++xq) {
                        // lane i addresses row (i % 8) + 8 ((i / 8) % 2) of piece 2 xq + i / 16
                        const int mi = lane >> 3, rr = lane & 7;
                        const int row = rr + 8 * (mi & 1), piece = 2 * xq + (mi >> 1);
                        uint32_t r4[4];
                        gm_ldsm4(tb + (m * 16 + row) * GM_TSTRIDE + piece * 16, r4);
                        aw[m][2 * xq][0] = r4[0];
                        aw[m][2 * xq][1] = r4[1];
                        aw[m][2 * xq + 1][0] = r4[2];
                        aw[m][2 * xq + 1][1] = r4[3];
                    }
                // the step's B fragments, all issued before the first mma
                uint32_t bf[NBLK][NTL][2];
#pragma unroll
                for (int kb = 0; kb < NBLK; ++kb) {
                    // record chunk of the mma's k = 0 .. 15
                    const int c = WB == 4 ? NBLK * sc + kb : (WB == 2 ? 4 * sc + (kb >> 1) : 4 * sc + 2 * kb);
#pragma unroll
                    for (int jj = 0; jj < NTL; ++jj) {
                        bf[kb][jj][0] = bf[kb][jj][1] = 0;
                        if (boff[jj] >= 0) {
                            if constexpr (WB == 4) {
                                const uint2 bb = *reinterpret_cast<const uint2 *>(sm + boff[jj] + ((t >> 1) * p.cpr + c) * 16 + (t & 1) * 8);
                                bf[kb][jj][0] = bb.x;
                                bf[kb][jj][1] = bb.y;
                            } else if constexpr (WB == 2) {
                                // digit words 4 t + 2 (kb & 1) and the next: piece t, 8 bytes in
                                const uint2 bb = *reinterpret_cast<const uint2 *>(sm + boff[jj] + (t * p.cpr + c) * 16 + (kb & 1) * 8);
                                bf[kb][jj][0] = bb.x;
                                bf[kb][jj][1] = bb.y;
                            } else {
                                bf[kb][jj][0] = *reinterpret_cast<const uint32_t *>(sm + boff[jj] + c * 16 + 4 * t);
                                bf[kb][jj][1] = *reinterpret_cast<const uint32_t *>(sm + boff[jj] + (c + 1) * 16 + 4 * t);
                            }
                        }
                    }
                }
#pragma unroll
                for (int kb = 0; kb < NBLK; ++kb) {
                    uint32_t a[NM][4];
#pragma unroll
                    for (int m = 0; m < NM; ++m) {
                        if constexpr (WB == 2) {
                            // word t of piece kb / 2, fields flipped to offset binary (code + 2):
                            // byte b of field pair (kb & 1) is codes 16 t + 4 b + 2 (kb & 1) and + 1
                            const int sh = 4 * (kb & 1);
                            const uint32_t wg = aw[m][kb >> 1][0] ^ 0xAAAAAAAAu, wh = aw[m][kb >> 1][1] ^ 0xAAAAAAAAu;
                            a[m][0] = (wg >> sh) & 0x03030303u;
                            a[m][1] = (wh >> sh) & 0x03030303u;
                            a[m][2] = (wg >> (sh + 2)) & 0x03030303u;
                            a[m][3] = (wh >> (sh + 2)) & 0x03030303u;
                        } else if constexpr (WB == 4) {
                            // two's-complement nibbles flipped to offset binary (code + 8)
                            const uint32_t wg = aw[m][kb][0] ^ 0x88888888u, wh = aw[m][kb][1] ^ 0x88888888u;
                            a[m][0] = wg & 0x0F0F0F0Fu;                    // codes 8t + 0, 2, 4, 6 of row g
                            a[m][1] = wh & 0x0F0F0F0Fu;                    // same of row g + 8
                            a[m][2] = (wg >> 4) & 0x0F0F0F0Fu;             // codes 8t + 1, 3, 5, 7
                            a[m][3] = (wh >> 4) & 0x0F0F0F0Fu;
                        } else {
                            a[m][0] = aw[m][2 * kb][0];
                            a[m][1] = aw[m][2 * kb][1];
                            a[m][2] = aw[m][2 * kb + 1][0];
                            a[m][3] = aw[m][2 * kb + 1][1];
                        }
                    }
                    const int c = WB == 4 ? NBLK * sc + kb : 4 * sc + 2 * kb;
                    const int blk = WB == 4 ? c : c >> 1;                        // Q8_0 block
#pragma unroll
                    for (int jj = 0; jj < NTL; ++jj) {
                        if constexpr (NDIG == 3) {
#pragma unroll
                            for (int m = 0; m < NM; ++m)
                                gm_mma(acc[m][jj], a[m][0], a[m][1], a[m][2], a[m][3], bf[kb][jj][0], bf[kb][jj][1], WB != 8);
                        } else {
                            // started from the block's offset correction, scaled by the token's d_b
                            int cr[2] = {0, 0};
                            float dq[2] = {0.f, 0.f};
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                if (coff[jj][h] >= 0) {
                                    dq[h] = reinterpret_cast<const float *>(sm + coff[jj][h])[blk];
                                    cr[h] = reinterpret_cast<const int *>(sm + coff[jj][h] + (RL.bytes - RL.hdr) / 2)[blk];
                                }
#pragma unroll
                            for (int m = 0; m < NM; ++m) {
                                int d4[4] = {cr[0], cr[1], cr[0], cr[1]};
                                gm_mma(d4, a[m][0], a[m][1], a[m][2], a[m][3], bf[kb][jj][0], bf[kb][jj][1], WB != 8);
#pragma unroll
                                for (int q = 0; q < 4; ++q) facc[m][jj][q] = fmaf(dq[q & 1], (float)d4[q], facc[m][jj][q]);
                            }
                        }
                    }
                }
            };
            if constexpr (RD) {
                // fixed point: the lane's own 16 bytes of rows g and g + 8 are its A
                // fragments (block 4 sc + t for int4, half block for int8); the
                // records give the matching digits, one step of loads ahead
                uint4 nx[NM][2];
                auto load = [&](int sc) {
                    if (sc < nsc)
#pragma unroll
                        for (int m = 0; m < NM; ++m) {
                            nx[m][0] = ld_stream16(wa[m] + (size_t)sc * GM_SCB);
                            nx[m][1] = ld_stream16(wb[m] + (size_t)sc * GM_SCB);
                        }
                };
                load(0);
#pragma unroll 1
                for (int sc = 0; sc < nsc; ++sc) {
                    uint32_t cw[NM][2][4];
#pragma unroll
                    for (int m = 0; m < NM; ++m)
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            cw[m][hf][0] = nx[m][hf].x;
                            cw[m][hf][1] = nx[m][hf].y;
                            cw[m][hf][2] = nx[m][hf].z;
                            cw[m][hf][3] = nx[m][hf].w;
                        }
                    load(sc + 1);
                    const int c = 4 * sc + t;                  // the record chunk of this lane's 16 bytes
                    // mma j: k = 4 t .. 4 t + 3 <- word j's low nibbles (int4) or word 2 j
                    // (int8); k = 16 + 4 t .. <- its high nibbles or word 2 j + 1
                    uint32_t bf[NBLK][NTL][2];
#pragma unroll
                    for (int j = 0; j < NBLK; ++j)
#pragma unroll
                        for (int jj = 0; jj < NTL; ++jj) {
                            bf[j][jj][0] = bf[j][jj][1] = 0;
                            if (boff[jj] >= 0) {
                                // int4: digit words 2 j, 2 j + 1; int2: 4 (j / 2) + 2 (j & 1) and the next
                                const int off = WB != 8 ? ((j >> 1) * p.cpr + c) * 16 + (j & 1) * 8 : c * 16 + 8 * j;
                                const uint2 bb = *reinterpret_cast<const uint2 *>(sm + boff[jj] + off);
                                bf[j][jj][0] = bb.x;
                                bf[j][jj][1] = bb.y;
                            }
                        }
#pragma unroll
                    for (int j = 0; j < NBLK; ++j) {
                        uint32_t a[NM][4];
#pragma unroll
                        for (int m = 0; m < NM; ++m) {
                            if constexpr (WB == 2) {
                                const int sh = 4 * (j & 1);
                                const uint32_t wg = cw[m][0][j >> 1] ^ 0xAAAAAAAAu, wh = cw[m][1][j >> 1] ^ 0xAAAAAAAAu;
                                a[m][0] = (wg >> sh) & 0x03030303u;
                                a[m][1] = (wh >> sh) & 0x03030303u;
                                a[m][2] = (wg >> (sh + 2)) & 0x03030303u;
                                a[m][3] = (wh >> (sh + 2)) & 0x03030303u;
                            } else if constexpr (WB == 4) {
                                const uint32_t wg = cw[m][0][j] ^ 0x88888888u, wh = cw[m][1][j] ^ 0x88888888u;
                                a[m][0] = wg & 0x0F0F0F0Fu;
                                a[m][1] = wh & 0x0F0F0F0Fu;
                                a[m][2] = (wg >> 4) & 0x0F0F0F0Fu;
                                a[m][3] = (wh >> 4) & 0x0F0F0F0Fu;
                            } else {
                                a[m][0] = cw[m][0][2 * j];
                                a[m][1] = cw[m][1][2 * j];
                                a[m][2] = cw[m][0][2 * j + 1];
                                a[m][3] = cw[m][1][2 * j + 1];
                            }
                        }
#pragma unroll
                        for (int jj = 0; jj < NTL; ++jj)
#pragma unroll
                            for (int m = 0; m < NM; ++m)
                                gm_mma(acc[m][jj], a[m][0], a[m][1], a[m][2], a[m][3], bf[j][jj][0], bf[j][jj][1], WB != 8);
                    }
                }
            } else {
                // the ring: GM_STAGES - 1 steps in flight ahead of the one computed
                __syncwarp();                                  // the last unit's tile reads are done
#pragma unroll
                for (int q = 0; q < GM_STAGES - 1; ++q) issue(q);
#pragma unroll 1
                for (int sc = 0; sc < nsc; ++sc) {
                    gm_wait_groups<GM_STAGES - 2>();           // this lane's copies of step sc have landed
                    __syncwarp();                              // ... and every lane's; tile (sc - 1) % S is free
                    issue(sc + GM_STAGES - 1);
                    step(sc);
                }
                gm_wait_groups<0>();
            }
            // ---- epilogue: accumulators -> the warp's tile as [m][row][column] -> outputs
            __syncwarp();
            float *stf = reinterpret_cast<float *>(tile);
            int *sti = reinterpret_cast<int *>(tile);
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int jj = 0; jj < NTL; ++jj)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int row = g + 8 * (q >> 1), col = 8 * jj + 2 * t + (q & 1);
                        if constexpr (NDIG == 3) sti[(m * 16 + row) * NC + col] = acc[m][jj][q];
                        else stf[(m * 16 + row) * NC + col] = facc[m][jj][q];
                    }
            __syncwarp();
            for (int q = lane; q < GM_ROWS * nt; q += 32) {
                const int row = q & (GM_ROWS - 1), tk = q >> 4;
                const int r = r0 + row;
                if (r >= p.rows) continue;
                float x[NM];
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    if constexpr (NDIG == 3) {
                        const int *pp = sti + (m * 16 + row) * NC + tk * 3;
                        const int *tt = tot + recidx(tk) * 4;
                        const int P0 = pp[0] - (WB != 8 ? tt[0] : 0), P1 = pp[1] - (WB != 8 ? tt[1] : 0),
                                  P2 = pp[2] - (WB != 8 ? tt[2] : 0);
                        const float sg = *reinterpret_cast<const float *>(recs + (size_t)recidx(tk) * p.rec_bytes + RL.hdr);
                        x[m] = sg * fmaf(65536.f, (float)P2, fmaf(256.f, (float)P1, (float)P0));
                    } else {
                        x[m] = stf[(m * 16 + row) * NC + tk];
                    }
                }
                const int64_t o = routed ? (int64_t)p0 + tk : p.sh_out_row0 + p0 + tk;
                QRX_CHECK_OR(o >= 0 && o < n_out, continue);
                const float s0 = routed ? p.m[0].s[(int64_t)e * p.m[0].ss + r] : p.msh[0].s[r];
                if constexpr (GATEUP) {
                    const float s1 = routed ? p.m[1].s[(int64_t)e * p.m[1].ss + r] : p.msh[1].s[r];
                    p.out[o * p.out_ld + r] = silu_mul(s0 * x[0], s1 * x[NM - 1]);
                } else {
                    p.out[o * p.out_ld + r] = s0 * x[0];
                }
            }
        }
    }
}

// ---------------------------------------------------------------- host side
struct GmPlan {
    G2P p;
    int ntl;
};

// Geometry for one projection (`nm` matrices of `rows` rows x K codes) of a call
// of T tokens: the n-tiles per pass (columns = tokens x planes, up to 24 for
// the fixed point and 32 for Q8_0 and as many as T needs), the slot table's
// capacity after splitting, and how many instances' records one phase holds.
static inline bool gm_plan(GmPlan &pl, int wbits, int ndig, int K, int rows, int nm, int T, int E, int k)
{
    G2P &p = pl.p;
    p = G2P{};
    if ((wbits != 4 && wbits != 8 && !(wbits == 2 && ndig == 3)) || T < 1 || T > 64 || rows < 1 || E < 1 || k < 1 ||
        k > 32)
        return false;
    p.K = K;
    p.rows = rows;
    p.row_bytes = K * wbits / 8;
    if (K % 32 || p.row_bytes % GM_SCB) return false;
    p.cpr = p.row_bytes / 16;
    p.rw = GM_ROWS;
    p.nwu = (rows + GM_ROWS - 1) / GM_ROWS;
    p.rec_bytes = (g2_rec(ndig, K, p.cpr).bytes + 127) & ~127;
    const int A = T * k;
    auto al = [](int v, int a) { return (v + a - 1) / a * a; };
    for (int ntl = ndig == 3 ? 3 : 4; ntl >= 1; --ntl) {
        if (ndig == 1 && ntl == 3) continue;
        const int ntok = ndig == 3 ? 8 * ntl / 3 : 8 * ntl;
        // no more n-tiles than the call's tokens need
        const int need = ndig == 3 ? (3 * T + 7) / 8 : (T + 7) / 8;
        if (ntl > 1 && ntl - 1 >= need && !(ndig == 1 && ntl == 4 && need > 2)) continue;
        p.ms = (E < A ? E : A) + 1 + (A + T + ntok - 1) / ntok + 1;
        const int ring = GM_STAGES * nm * GM_ROWS * GM_TSTRIDE, stage = nm * GM_ROWS * 8 * ntl * 4;
        p.ntile = al(ring > stage ? ring : stage, 16);
        int o = 0;
        p.o_sl = o;
        o = al(o + (4 + 3 * p.ms) * 4, 16);
        p.o_srt = o;
        o = al(o + A * 4, 16);
        p.o_pre = o;
        o = al(o + (p.ms + 1) * 8, 16);
        p.o_seg = o;
        o = al(o + (1 + 3 * p.ms) * 4, 16);
        p.o_hmx = o;                                   // warp tiles
        o = al(o + G2_NW * p.ntile, 16);
        const int per = ntok * (p.rec_bytes + 16 + G2_NW * 4);
        p.allrec = nm == 2 && T <= ntok;               // gate/up: every token's record, once
        if (p.allrec) {
            p.slot_cap = p.ms;
            p.nrec = T;
        } else {
            int cap = (G2_SMEM_MAX - 256 - o) / per;
            if (cap > p.ms) cap = p.ms;
            if (cap < 1) continue;
            p.slot_cap = cap;
            p.nrec = cap * ntok;
        }
        p.o_route = o;                                 // plane digit totals
        o = al(o + p.nrec * 16, 16);
        p.o_rmax = o;
        o = al(o + p.nrec * G2_NW * 4, 128);
        p.o_rec = o;
        o += p.nrec * p.rec_bytes;
        p.smem = o;
        if (o > G2_SMEM_MAX) continue;
        pl.ntl = ntl;
        return true;
    }
    return false;
}

template <int WB, int ND, int NTL, bool GU>
static cudaError_t gm_go(const G2P &p, int grid, cudaStream_t st)
{
    auto kern = k_gmma<WB, ND, NTL, GU>;
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

template <bool GU>
static cudaError_t gm_dispatch(const GmPlan &pl, int wbits, int ndig, int grid, cudaStream_t st)
{
#define QRX_GM(WB, ND, NTL) \
    if (wbits == WB && ndig == ND && pl.ntl == NTL) return gm_go<WB, ND, NTL, GU>(pl.p, grid, st);
    QRX_GM(4, 3, 1) QRX_GM(4, 3, 2) QRX_GM(4, 3, 3) QRX_GM(4, 1, 1) QRX_GM(4, 1, 2) QRX_GM(4, 1, 4)
    QRX_GM(8, 3, 1) QRX_GM(8, 3, 2) QRX_GM(8, 3, 3) QRX_GM(8, 1, 1) QRX_GM(8, 1, 2) QRX_GM(8, 1, 4)
    QRX_GM(2, 3, 1) QRX_GM(2, 3, 2) QRX_GM(2, 3, 3)
#undef QRX_GM
    return cudaErrorInvalidValue;
}

bool gm_use(const FfnArgs &a)
{
    if (a.T < 2 || a.T > 64) return false;
    GmPlan pg, pd;
    return gm_plan(pg, a.wbits, g2_ndig(a), a.H, a.I, 2, a.T, a.E, a.k) &&
           gm_plan(pd, a.wbits, g2_ndig(a), a.I, a.H, 1, a.T, a.E, a.k);
}

cudaError_t launch_gm_gateup(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = g2_ndig(a);
    GmPlan pl;
    if (!gm_plan(pl, a.wbits, ndig, a.H, a.I, 2, a.T, a.E, a.k)) return cudaErrorInvalidValue;
    g2_gateup_args(pl.p, a, nullptr);
    return gm_dispatch<true>(pl, a.wbits, ndig, num_sms, st);
}

cudaError_t launch_gm_down(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int ndig = g2_ndig(a);
    GmPlan pl;
    if (!gm_plan(pl, a.wbits, ndig, a.I, a.H, 1, a.T, a.E, a.k)) return cudaErrorInvalidValue;
    g2_down_args(pl.p, a, nullptr);
    return gm_dispatch<false>(pl, a.wbits, ndig, num_sms, st);
}

}  // namespace qrx
