// k_ffn_tc.cuh -- expert FFN over the batch union as grouped GEMMs on the
// tcgen05 tensor cores, for batches with many tokens per expert (prefill,
// long verify batches) and bf16 activations.
//
// README "JustVugg/colibri", section "已实现的功能": batch-union MoE (each
// unique expert of a batch is read once and applied to all positions routed
// to it); packed int4 weights with per-row scales, dequantised on use.  With
// ~100 tokens per expert the work is a dense contraction, so it runs on the
// tensor cores: int4 codes are exact in bf16, products accumulate in f32, and
// the per-row scale multiplies the accumulator in the epilogue.
//
// Tiles.  A work item is (slot, 256 weight rows, up to 128 tokens): the
// weights are the MMA's M side (two M=128 halves sharing one B tile: for
// gate/up 128 rows of the gate matrix and the same 128 rows of the up matrix,
// for down 256 consecutive rows) and the tokens its N side; K advances in stages of 64 (one 128-byte swizzle atom of
// bf16).  B is always a run of consecutive rows of one bf16 matrix: for
// gate/up the tokens gathered into expert order by k_gather_x, for down the
// rows of h that gate/up wrote in the same order.  Roles per CTA (one CTA per
// SM, persistent over items):
//   warp 0      TMA producer: the packed int4 rows of the item, 128 bytes
//               (4 k-stages) per row at a time, into a 128B-swizzled "raw"
//               stage, after an L2 prefetch of the same box issued TC_PF raw
//               stages earlier; the token rows of each k-stage into its B tile;
//   warp 1      allocates 512 TMEM columns (two 256x128 f32 accumulators) and
//               issues tcgen05.mma (M=128, N<=128, K=16; two halves x four
//               per stage); each stage is released with tcgen05.commit to its
//               "empty" mbarrier, each finished item with a commit to its
//               accumulator's "full";
//   warps 4-7   epilogue: tcgen05.ld of the accumulator, row scales, SwiGLU
//               (gate/up) or the output rows (down), stores;
//   8 warps     dequantisers (2, 3, 8, 10, 11, 12, 14, 15): thread r turns
//               row r's 64 codes of the stage into bf16 in the 128B-swizzled
//               K-major A tile.
// One thread issues the MMAs: the tensor core's queue is only a few
// instructions deep, so everything that thread does between two stages (its
// barrier checks, the commit) is time the tensor core may sit idle; the other
// roles that wait long (producer, epilogue) sleep between polls.
// Dequantisation writes the 8 codes of a packed word in the order
// (0,4,1,5,2,6,3,7); the token rows (and h for the down projection) are kept
// in the same order within every 8-element chunk, so the contraction is
// unchanged.  All mbarrier waits are bounded; a timeout raises the device
// status flag, every role leaves its loops, the producer waits (bounded) for
// the copies it started, and only then is TMEM freed.
#pragma once
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "qrx_dev.cuh"
#include "qrx_check.cuh"

namespace qrx {

constexpr int TC_HALF = 128;                 // rows per MMA (M)
constexpr int TC_M = 2 * TC_HALF;            // weight rows per item
constexpr int TC_BK = 64;                    // K per stage
constexpr int TC_RK = 4;                     // stages per raw (int4) stage: 128 bytes of a row
constexpr int TC_NMAX = 128;                 // tokens per item
constexpr int TC_S = 3;                      // stages of (bf16 A tile, B tile)
constexpr int TC_RS = 2;                     // raw stages (int4 rows from HBM)
constexpr int TC_PF = 4;                     // raw stages prefetched into L2 ahead of their copy
constexpr int TC_BOX_ROWS = 32;              // token rows per B copy
constexpr int TC_A_BYTES = TC_M * 128;       // bf16 A tile (two halves), 32 KB
constexpr int TC_B_BYTES = TC_NMAX * 128;    // bf16 B tile, 16 KB
constexpr int TC_RAW_BYTES = TC_M * 128;     // int4 rows, 4 stages, 32 KB
// Warp roles.  Warp w issues from SM sub-partition w % 4, and the MMA thread
// runs a serial chain (barrier checks, descriptors, MMAs, commit) that loses
// every issue arbitration against busy warps: its sub-partition (1) holds only
// the MMA warp, one epilogue warp (asleep between items) and two idle warps,
// while the eight dequantiser warps share sub-partitions 0, 2 and 3.
constexpr int TC_PRODUCER = 0, TC_MMA = 1, TC_EPI0 = 4;  // epilogue: warps 4..7 (TMEM quarter = warp % 4)
constexpr int TC_DQ_WARPS = 8;
constexpr int TC_THREADS = 16 * 32;                      // warps 9 and 13 idle
// dequantiser index of warp w (-1: not a dequantiser): warps 2, 3, 8, 10, 11, 12, 14, 15
__host__ __device__ constexpr int tc_dq_index(int w)
{
    return w == 2 ? 0 : w == 3 ? 1 : w == 8 ? 2 : w == 10 ? 3 : w == 11 ? 4 : w == 12 ? 5 : w == 14 ? 6
         : w == 15 ? 7 : -1;
}
#ifndef TC_BS
#define TC_BS 16                              // mbarrier spacing in 8-byte words: one per 128-byte line
#endif
constexpr int TC_NBARS = 3 * TC_S + 2 * TC_RS + 5;   // + acc_full[2], acc_empty[2], drain
constexpr int TC_CTL_BYTES = (TC_NBARS + 1) * TC_BS * 8;
// dynamic shared memory: 1024-byte alignment slack, the stages, barriers and
// flags, the item prefix over up to maxslots slots
__host__ __device__ constexpr int tc_smem_bytes(int maxslots)
{
    return 1024 + TC_S * (TC_A_BYTES + TC_B_BYTES) + TC_RS * TC_RAW_BYTES + TC_CTL_BYTES +
           (maxslots + 2) * 8;
}

// Position p within an 8-element chunk holds element tc_perm(p).
__host__ __device__ constexpr int tc_perm(int p) { return (p & 1) ? 4 + (p >> 1) : (p >> 1); }
__host__ __device__ constexpr int tc_inv_perm(int e) { return e < 4 ? 2 * e : 2 * (e - 4) + 1; }

struct TcP {
    int rows, K, mtiles, kstages;     // rows per matrix (gate/up: I, down: H)
    int half_rows;                    // row offset of half 1 within an item (gate/up: 0, down: 128)
    const float *s[2];                // routed row scales of half 0 / 1's matrix, expert stride s_stride
    int64_t s_stride[2];
    const float *s_sh[2];
    int routed, shared, E, k, T;
    const int32_t *offsets, *union_ids, *n_union;
    int64_t b_sh_row0;           // B row of the shared expert's first token
    float *out;                  // gate/up: h f32 [rows of positions][I] (may be null); down: y f32
    int64_t out_ld, sh_out_row0;
    __nv_bfloat16 *hperm;        // gate/up: h bf16 chunk-permuted [positions][I] (may be null)
    int gateup;
};

__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr)
{
    // K-major, 128-byte swizzle: 8-row groups 1024 B apart (SBO), version 1.
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint32_t tc_idesc(int N)
{
    // D f32, A bf16, B bf16, both K-major, N >> 3, M >> 4.
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(TC_HALF >> 4) << 24);
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_expect(uint32_t mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes)
                 : "memory");
}

// Tiled TMA loads (no multicast) completing on `mbar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                            uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(mbar)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

// Item geometry for slot s: token tiles of at most 128, balanced, multiple of 16.
struct TcSlot {
    int ntok, ntiles, nbase;
};

__device__ __forceinline__ TcSlot tc_slot(const TcP &p, int s, int nu)
{
    TcSlot r;
    if (s < nu) {
        const int e = p.union_ids[s];
        r.ntok = (e >= 0 && e < p.E) ? p.offsets[e + 1] - p.offsets[e] : 0;
    } else {
        r.ntok = p.T;
    }
    r.ntiles = (r.ntok + TC_NMAX - 1) / TC_NMAX;
    const int per = r.ntiles ? (r.ntok + r.ntiles - 1) / r.ntiles : 0;
    r.nbase = (per + 15) / 16 * 16;
    return r;
}

// One work item, decoded from its index through the item prefix over slots.
struct TcItem {
    int slot, mt, n0, nv, nn, e;
    bool routed;
    int64_t b0;             // first B row
};

__device__ __forceinline__ TcItem tc_decode(const TcP &p, const int64_t *pre, int nslots, int nu,
                                            int64_t it)
{
    int lo = 0, hi = nslots;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= it) lo = mid; else hi = mid;
    }
    TcItem d;
    d.slot = lo;
    const TcSlot sl = tc_slot(p, lo, nu);
    const int64_t r = it - pre[lo];
    const int ni = (int)(r / p.mtiles);
    d.mt = (int)(r % p.mtiles);
    d.n0 = ni * sl.nbase;
    d.nv = min(sl.nbase, sl.ntok - d.n0);
    d.nn = sl.nbase;
    d.routed = lo < nu;
    d.e = 0;
    int64_t p0 = p.b_sh_row0;
    if (d.routed) {
        const int e = p.union_ids[lo];
        d.e = (e >= 0 && e < p.E) ? e : 0;
        p0 = p.offsets[d.e];
    }
    d.b0 = p0 + d.n0;
    return d;
}

// Bounded wait that also gives up (false, no new status) once another role
// has raised the abort flag; on its own timeout it raises both.  Roles off
// the MMA's critical path (park = true) are parked by the barrier itself: each
// try_wait carries a suspend-time hint, so the warp sleeps until the phase
// completes (or the hint runs out) and leaves the issue slots of its SM
// sub-partition to the warps that work.  The MMA thread polls (park = false).
constexpr uint32_t TC_PARK_NS = 1000;          // suspend hint of a parked poll
constexpr long long TC_PARK_CAP = 1ll << 21;   // parked polls before a wait gives up

__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                        bool park = false)
{
    const uint32_t a = smem_u32(bar);
    for (long long it = 0; it < (park ? TC_PARK_CAP : GV_WAIT_CAP); ++it) {
        uint32_t done;
        if (park)
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(done)
                : "r"(a), "r"(parity), "r"(TC_PARK_NS)
                : "memory");
        else
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(done)
                : "r"(a), "r"(parity)
                : "memory");
        if (done) return true;
        if ((park || (it & 255) == 255) && *abort_flag) return false;
    }
    *abort_flag = 1;
    raise_status(DERR_TIMEOUT);
    return false;
}

// tc_wait with a one-instruction fast path for a phase that has already
// completed (the common case on the MMA thread).
__device__ __forceinline__ bool tc_wait_fast(uint64_t *bar, uint32_t parity, volatile int *abort_flag)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done ? true : tc_wait(bar, parity, abort_flag);
}

// One tcgen05.mma (kind::f16, cta_group::1): D[tmem] (+)= A[smem] * B[smem].
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred pd;\n\t"
        "setp.ne.b32 pd, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pd;\n\t}" ::"r"(d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

// tc_wait for a whole warp: lane 0 polls (one shared-memory request per poll
// instead of 32) and broadcasts the outcome.
__device__ __forceinline__ bool tc_wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             bool park = false)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = tc_wait(bar, parity, abort_flag, park) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// First weight row of half `hf` of row tile mt (gate/up: both halves start at
// mt*128 of their own matrix; down: mt*256 and mt*256 + 128 of one matrix).
__device__ __forceinline__ int tc_row0(const TcP &p, int mt, int hf)
{
    return p.half_rows ? mt * TC_M + hf * TC_HALF : mt * TC_HALF;
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    k_ffn_tc(const __grid_constant__ CUtensorMap mw0, const __grid_constant__ CUtensorMap mw1,
             const __grid_constant__ CUtensorMap msh0, const __grid_constant__ CUtensorMap msh1,
             const __grid_constant__ CUtensorMap mb, const TcP p)
{
    extern __shared__ __align__(1024) unsigned char tsm_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *tsm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sA = tsm;                                   // [S][256 rows][128 B]
    unsigned char *sB = sA + TC_S * TC_A_BYTES;                // [S][128 rows][128 B]
    unsigned char *sR = sB + TC_S * TC_B_BYTES;                // [RS][256 rows][128 B]
    unsigned char *ctl = sR + TC_RS * TC_RAW_BYTES;
    // barriers TC_BS words apart (each on its own 128-byte line at the default)
    uint64_t *full_a = reinterpret_cast<uint64_t *>(ctl);      // [S]  dequantisers
    uint64_t *full_b = full_a + TC_S * TC_BS;                  // [S]  B copies
    uint64_t *empty = full_b + TC_S * TC_BS;                   // [S]  MMA done with the stage
    uint64_t *raw_full = empty + TC_S * TC_BS;                 // [RS] int4 copies
    uint64_t *raw_empty = raw_full + TC_RS * TC_BS;            // [RS] dequantisers done
    uint64_t *acc_full = raw_empty + TC_RS * TC_BS;            // [2]
    uint64_t *acc_empty = acc_full + 2 * TC_BS;                // [2]
    uint64_t *drain = acc_empty + 2 * TC_BS;                   // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + TC_BS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int64_t *pre = reinterpret_cast<int64_t *>(ctl + TC_CTL_BYTES);   // [nslots + 1] item prefix

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    const int nu = p.routed ? *p.n_union : 0;
    const int nslots = nu + (p.shared ? 1 : 0);

    if (tid == 0) {
        for (int i = 0; i < TC_S; ++i) {
            mbar_init(smem_u32(&full_a[(i) * TC_BS]), TC_DQ_WARPS);
            mbar_init(smem_u32(&full_b[(i) * TC_BS]), 1);
            mbar_init(smem_u32(&empty[(i) * TC_BS]), 1);
        }
        for (int i = 0; i < TC_RS; ++i) {
            mbar_init(smem_u32(&raw_full[(i) * TC_BS]), 1);
            mbar_init(smem_u32(&raw_empty[(i) * TC_BS]), TC_DQ_WARPS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&acc_full[(i) * TC_BS]), 1);
            mbar_init(smem_u32(&acc_empty[(i) * TC_BS]), 4);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == TC_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // item prefix over slots: items of slot s = ntiles * mtiles
    if (warp == TC_EPI0) {
        int64_t run = 0;
        for (int s0 = 0; s0 < nslots; s0 += 32) {
            const int s = s0 + lane;
            int64_t cnt = 0;
            if (s < nslots) cnt = (int64_t)tc_slot(p, s, nu).ntiles * p.mtiles;
            int64_t inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (s < nslots) pre[s] = run + inc - cnt;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pre[nslots] = run;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const int64_t nitems = pre[nslots];

    if (warp == TC_PRODUCER) {
        // ================= TMA producer (one thread) =================
        if (lane == 0) {
            uint32_t g = 0, rg = 0;
            bool ok = true;
            // L2 prefetch cursor, TC_PF raw stages ahead of the copies
            const int kraw = p.kstages / TC_RK;
            int64_t pf_it = blockIdx.x;
            int pf_kr = 0;
            TcItem pf_d{};
            if (pf_it < nitems) pf_d = tc_decode(p, pre, nslots, nu, pf_it);
            auto pf_step = [&]() {
                if (pf_it >= nitems) return;
                const int zz = pf_d.routed ? pf_d.e : 0;
                tma_prefetch_3d(pf_d.routed ? &mw0 : &msh0, pf_kr * 128, tc_row0(p, pf_d.mt, 0), zz);
                tma_prefetch_3d(pf_d.routed ? &mw1 : &msh1, pf_kr * 128, tc_row0(p, pf_d.mt, 1), zz);
                if (++pf_kr == kraw) {
                    pf_kr = 0;
                    pf_it += gridDim.x;
                    if (pf_it < nitems) pf_d = tc_decode(p, pre, nslots, nu, pf_it);
                }
            };
            for (int i = 0; i < TC_PF; ++i) pf_step();
            for (int64_t it = blockIdx.x; ok && it < nitems && !*abort_flag; it += gridDim.x) {
                const TcItem d = tc_decode(p, pre, nslots, nu, it);
                const CUtensorMap *wm0 = d.routed ? &mw0 : &msh0;
                const CUtensorMap *wm1 = d.routed ? &mw1 : &msh1;
                const int z = d.routed ? d.e : 0;
                const int nbox = (d.nn + TC_BOX_ROWS - 1) / TC_BOX_ROWS;
                for (int kb = 0; kb < p.kstages; ++kb) {
                    if (kb % TC_RK == 0) {
                        const uint32_t rs = rg % TC_RS;
                        if (rg >= TC_RS && !tc_wait(&raw_empty[(rs) * TC_BS], ((rg / TC_RS) - 1) & 1, abort_flag, true)) {
                            ok = false;
                            break;
                        }
                        pf_step();
                        const uint32_t dst = smem_u32(sR + rs * TC_RAW_BYTES);
                        const uint32_t bar = smem_u32(&raw_full[(rs) * TC_BS]);
                        mbar_expect(bar, TC_RAW_BYTES);
                        tma_load_3d(dst, wm0, (kb / TC_RK) * 128, tc_row0(p, d.mt, 0), z, bar);
                        tma_load_3d(dst + TC_RAW_BYTES / 2, wm1, (kb / TC_RK) * 128, tc_row0(p, d.mt, 1), z,
                                    bar);
                        ++rg;
                    }
                    const uint32_t sb = g % TC_S;
                    if (g >= TC_S && !tc_wait(&empty[(sb) * TC_BS], ((g / TC_S) - 1) & 1, abort_flag, true)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = smem_u32(&full_b[(sb) * TC_BS]);
                    mbar_expect(bar, (uint32_t)(nbox * TC_BOX_ROWS * 128));
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d(smem_u32(sB + sb * TC_B_BYTES + j * TC_BOX_ROWS * 128), &mb, kb * TC_BK,
                                    (int)(d.b0 + j * TC_BOX_ROWS), bar);
                    ++g;
                }
            }
            // the copies started above land before the CTA may leave: wait for
            // the last phase armed on every barrier (already complete unless a
            // consumer gave up)
            for (uint32_t i = 0; i < (uint32_t)TC_S && i < g; ++i) {
                const uint32_t n = (g - 1 - i) / TC_S + 1;
                if (!mbar_wait(smem_u32(&full_b[(i) * TC_BS]), (n - 1) & 1)) raise_status(DERR_TIMEOUT);
            }
            for (uint32_t i = 0; i < (uint32_t)TC_RS && i < rg; ++i) {
                const uint32_t n = (rg - 1 - i) / TC_RS + 1;
                if (!mbar_wait(smem_u32(&raw_full[(i) * TC_BS]), (n - 1) & 1)) raise_status(DERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == TC_MMA) {
        // ================= MMA issue (one thread) =================
        // The tensor core takes the next MMA only when its short queue has
        // room, and each issue already costs tens of cycles, so the issuing
        // thread runs a minimal chain: descriptors of stage 0 computed once and
        // moved by constants, stage/phase counters kept incrementally, one
        // try_wait per barrier when the phase has completed, one commit.
        if (lane == 0) {
            const uint64_t dA0 = tc_desc_sw128(smem_u32(sA)), dB0 = tc_desc_sw128(smem_u32(sB));
            uint32_t st = 0, ph = 0;              // ring position, carried across items
            uint64_t da = dA0, db = dB0;          // descriptors of stage st
            int local = 0;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < nitems && !*abort_flag; it += gridDim.x, ++local) {
                const TcItem d = tc_decode(p, pre, nslots, nu, it);
                const int a = local & 1;
                if (local >= 2 && !tc_wait(&acc_empty[(a) * TC_BS], ((local >> 1) - 1) & 1, abort_flag)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t d0 = tmem + (uint32_t)(a * 2 * TC_NMAX), d1 = d0 + TC_NMAX;
                const uint32_t idesc = tc_idesc(d.nn);
                for (int kb = 0; kb < p.kstages; ++kb) {
                    if (!tc_wait_fast(&full_b[(st) * TC_BS], ph, abort_flag) || !tc_wait_fast(&full_a[(st) * TC_BS], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t first = kb > 0 ? 1u : 0u;
                    // descriptor units are 16 bytes: K step of 16 bf16 = 2, half of A = 1024
                    tc_mma(d0, da, db, idesc, first);
                    tc_mma(d0, da + 2, db + 2, idesc, 1u);
                    tc_mma(d0, da + 4, db + 4, idesc, 1u);
                    tc_mma(d0, da + 6, db + 6, idesc, 1u);
                    tc_mma(d1, da + 1024, db, idesc, first);
                    tc_mma(d1, da + 1026, db + 2, idesc, 1u);
                    tc_mma(d1, da + 1028, db + 4, idesc, 1u);
                    tc_mma(d1, da + 1030, db + 6, idesc, 1u);
                    tc_commit(smem_u32(&empty[(st) * TC_BS]));
                    if (++st == TC_S) {
                        st = 0;
                        ph ^= 1u;
                        da = dA0;
                        db = dB0;
                    } else {
                        da += TC_A_BYTES >> 4;
                        db += TC_B_BYTES >> 4;
                    }
                }
                if (ok) tc_commit(smem_u32(&acc_full[(a) * TC_BS]));
            }
            // every MMA issued above has completed before TMEM is freed
            tc_commit(smem_u32(drain));
            if (!mbar_wait(smem_u32(drain), 0u)) raise_status(DERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp >= TC_EPI0 && warp < TC_EPI0 + 4) {
        // ================= epilogue (warps 4..7) =================
        const int q4 = warp & 3;                   // TMEM lane quarter of this warp
        QRX_CHECK_ONLY(const int64_t n_out = max(p.routed ? (int64_t)p.T * p.k : (int64_t)0, p.shared ? p.sh_out_row0 + p.T : (int64_t)0);)
        int local = 0;
        for (int64_t it = blockIdx.x; it < nitems && !*abort_flag; it += gridDim.x, ++local) {
            const TcItem d = tc_decode(p, pre, nslots, nu, it);
            // this thread's row of each half, and that row's scale
            const int r0 = tc_row0(p, d.mt, 0) + q4 * 32 + lane, r1 = tc_row0(p, d.mt, 1) + q4 * 32 + lane;
            const float *sb0 = d.routed ? p.s[0] + (int64_t)d.e * p.s_stride[0] : p.s_sh[0];
            const float *sb1 = d.routed ? p.s[1] + (int64_t)d.e * p.s_stride[1] : p.s_sh[1];
            const float sc0 = sb0[r0], sc1 = sb1[r1];
            const int64_t orow0 = d.routed ? d.b0 : p.sh_out_row0 + d.n0;
            const int a = local & 1;
            if (!tc_wait_warp(&acc_full[(a) * TC_BS], (local >> 1) & 1, abort_flag, true)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // 32 accumulator columns (tokens c0..c0+31) of half hf for this thread's row
            auto ld32 = [&](int hf, int c0, uint32_t (&v)[32]) {
                const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) +
                                       (uint32_t)(a * 2 * TC_NMAX + hf * TC_NMAX + c0);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
                    "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                      "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                      "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
                      "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
                      "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
                      "=r"(v[31])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            };
            if (p.gateup) {
                // half 0 holds gate row r0, half 1 the up row of the same index
#pragma unroll 1
                for (int c0 = 0; c0 < d.nn; c0 += 32) {
                    uint32_t vg[32], vu[32];
                    ld32(0, c0, vg);
                    ld32(1, c0, vu);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = c0 + j;
                        if (n >= d.nv) continue;
                        const int64_t orow = orow0 + n;
                        QRX_CHECK_OR(orow >= 0 && orow < n_out, continue);
                        const float h = silu_mul(sc0 * __uint_as_float(vg[j]), sc1 * __uint_as_float(vu[j]));
                        if (p.out) p.out[orow * p.out_ld + r0] = h;
                        if (p.hperm)
                            p.hperm[orow * p.rows + (r0 & ~7) + tc_inv_perm(r0 & 7)] = __float2bfloat16_rn(h);
                    }
                }
            } else {
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    const int rowg = hf ? r1 : r0;
                    const float sc = hf ? sc1 : sc0;
#pragma unroll 1
                    for (int c0 = 0; c0 < d.nn; c0 += 32) {
                        uint32_t v[32];
                        ld32(hf, c0, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int n = c0 + j;
                            if (n >= d.nv) continue;
                            const int64_t orow = orow0 + n;
                            QRX_CHECK_OR(orow >= 0 && orow < n_out, continue);
                            p.out[orow * p.out_ld + rowg] = sc * __uint_as_float(v[j]);
                        }
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[(a) * TC_BS]));
        }
    } else if (tc_dq_index(warp) >= 0) {
        // ================= dequantisers: thread r owns row r =================
        const int r = tc_dq_index(warp) * 32 + lane;
        const int hf = r >> 7, rr = r & 127, sw = rr & 7;
        const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
        uint32_t g = 0, rg = 0;
        bool ok = true;
        for (int64_t it = blockIdx.x; ok && it < nitems && !*abort_flag; it += gridDim.x) {
            for (int kb = 0; kb < p.kstages; ++kb) {
                const uint32_t rs = rg % TC_RS;
                if (kb % TC_RK == 0 && !tc_wait_warp(&raw_full[(rs) * TC_BS], (rg / TC_RS) & 1, abort_flag, true)) {
                    ok = false;
                    break;
                }
                const uint32_t st = g % TC_S;
                if (g >= TC_S && !tc_wait_warp(&empty[(st) * TC_BS], ((g / TC_S) - 1) & 1, abort_flag, true)) {
                    ok = false;
                    break;
                }
                // this row's 32 bytes of the stage: 16-byte chunks 2*sub and 2*sub+1
                const unsigned char *rrow = sR + rs * TC_RAW_BYTES + hf * (TC_RAW_BYTES / 2) + rr * 128;
                const int sub = kb % TC_RK;
                const uint4 r0 = *reinterpret_cast<const uint4 *>(rrow + (((2 * sub) ^ sw) << 4));
                const uint4 r1 = *reinterpret_cast<const uint4 *>(rrow + (((2 * sub + 1) ^ sw) << 4));
                const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                unsigned char *arow = sA + st * TC_A_BYTES + hf * (TC_A_BYTES / 2) + rr * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // two's-complement nibble -> offset binary -> bf16 (128 + code + 8) - 136
                    const uint32_t o = words[j] ^ 0x88888888u;
                    uint32_t q[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t v = ((o >> (4 * h)) & 0x000F000Fu) | 0x43004300u;
                        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v);
                        b = __hsub2(b, off);
                        q[h] = *reinterpret_cast<uint32_t *>(&b);
                    }
                    *reinterpret_cast<uint4 *>(arow + ((j ^ sw) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&full_a[(st) * TC_BS]));
                ++g;
                if (sub == TC_RK - 1) {
                    if (lane == 0) mbar_arrive(smem_u32(&raw_empty[(rs) * TC_BS]));
                    ++rg;
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == TC_MMA) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// B rows for gate/up: row r < A is the token of sorted assignment r, rows
// A..A+T-1 are the tokens in order (shared expert); each row chunk-permuted.
__global__ void __launch_bounds__(256) k_gather_x(const __nv_bfloat16 *__restrict__ x, int T, int H,
                                                  const int32_t *__restrict__ sorted, int64_t A, int k,
                                                  int64_t rows, __nv_bfloat16 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int chunks = H / 8;
    if (id >= rows * chunks) return;
    const int64_t r = id / chunks;
    const int c = (int)(id % chunks);
    int64_t t = r - A;
    if (r < A) {
        const int32_t a = sorted[r];
        QRX_CHECK_OR(a >= 0 && a < A, (void)0);      // an invalid position is zero-filled
        t = (a >= 0 && a < A) ? a / k : -1;
    }
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0 && t < T) v = reinterpret_cast<const uint4 *>(x + t * H)[c];
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&v);
    __nv_bfloat16 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = e[tc_perm(q)];
    reinterpret_cast<uint4 *>(out)[id] = *reinterpret_cast<const uint4 *>(o);
}

// h (f32 rows, stride ld) -> bf16 chunk-permuted rows.
__global__ void __launch_bounds__(256) k_perm_f32(const float *__restrict__ h, int64_t ld, int64_t rows,
                                                  int K, __nv_bfloat16 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int chunks = K / 8;
    if (id >= rows * chunks) return;
    const int64_t r = id / chunks;
    const int c = (int)(id % chunks);
    const float *src = h + r * ld + c * 8;
    __nv_bfloat16 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = __float2bfloat16_rn(src[tc_perm(q)]);
    reinterpret_cast<uint4 *>(out)[id] = *reinterpret_cast<const uint4 *>(o);
}

// ---------------------------------------------------------------- host side
constexpr int TC_MIN_T = 256;   // tokens from which the tensor-core path is used

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

// Packed weight rows of nexp experts: u8 [nexp][rows][row_bytes]; box 128 B x 128 rows.
static bool tc_map_weights(CUtensorMap *m, const void *w, int row_bytes, int rows, int nexp, int64_t stride)
{
    const auto fn = tc_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)nexp};
    const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)stride};
    const cuuint32_t box[3] = {128, (cuuint32_t)TC_HALF, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(w), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 rows [nrows][K]; box 64 elements x 32 rows.
static bool tc_map_rows(CUtensorMap *m, const void *b, int K, int64_t nrows)
{
    const auto fn = tc_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)nrows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)TC_BK, (cuuint32_t)TC_BOX_ROWS};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(b), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_shape_ok(int afmt, int wbits, int64_t T, int64_t H, int64_t I)
{
    return afmt == QRX_A_BF16 && wbits == 4 && T >= TC_MIN_T && H % (TC_BK * TC_RK) == 0 &&
           I % (TC_BK * TC_RK) == 0 && H % TC_M == 0 && I % TC_HALF == 0 && tc_encode_fn() != nullptr;
}

bool ffn_use_tc(const FfnArgs &a)
{
    return tc_shape_ok(a.afmt, a.wbits, a.T, a.H, a.I) && a.xperm && a.hperm;
}

// Weight maps: half 0 / 1 of every item read routed matrices m0 / m1 (gate and
// up, or down twice) and the shared expert's sh0 / sh1.
static cudaError_t tc_go(TcP &p, const MatRef &m0, const MatRef &m1, const MatRef &sh0, const MatRef &sh1,
                         const void *b, int64_t brows, int num_sms, cudaStream_t st, int maxslots)
{
    p.mtiles = p.half_rows ? p.rows / TC_M : p.rows / TC_HALF;
    p.kstages = p.K / TC_BK;
    const int row_bytes = p.K / 2;
    // zeroed: a launch without one expert set leaves its maps unused
    CUtensorMap mw0{}, mw1{}, msh0{}, msh1{}, mb{};
    bool ok = true;
    if (p.routed) {
        ok = ok && tc_map_weights(&mw0, m0.q, row_bytes, p.rows, p.E, m0.sq);
        ok = ok && tc_map_weights(&mw1, m1.q, row_bytes, p.rows, p.E, m1.sq);
    }
    if (p.shared) {
        ok = ok && tc_map_weights(&msh0, sh0.q, row_bytes, p.rows, 1, (int64_t)p.rows * row_bytes);
        ok = ok && tc_map_weights(&msh1, sh1.q, row_bytes, p.rows, 1, (int64_t)p.rows * row_bytes);
    }
    if (!p.routed) {
        mw0 = msh0;
        mw1 = msh1;
    }
    if (!p.shared) {
        msh0 = mw0;
        msh1 = mw1;
    }
    ok = ok && tc_map_rows(&mb, b, p.K, brows);
    if (!ok) return cudaErrorInvalidValue;
    const int smem = tc_smem_bytes(maxslots);
    if (smem > GV_SMEM_MAX) return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> configured{0};   // bit per device: max dynamic smem set
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !(configured.load(std::memory_order_acquire) >> dev & 1ull)) {
        err = cudaFuncSetAttribute(k_ffn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM_MAX);
        if (err != cudaSuccess) return err;
        if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
    }
    return launch_k(k_ffn_tc, dim3(num_sms), dim3(TC_THREADS), (size_t)smem, st, mw0, mw1, msh0, msh1, mb, p);
}

static void tc_common(TcP &p, const FfnArgs &a)
{
    p.routed = a.routed;
    p.shared = a.shared;
    p.E = a.E;
    p.k = a.k;
    p.T = a.T;
    p.offsets = a.offsets;
    p.union_ids = a.union_ids;
    p.n_union = a.n_union;
}

cudaError_t launch_ffn_tc_gateup(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    const int64_t A = a.routed ? (int64_t)a.T * a.k : 0;
    const int64_t rows = A + (a.shared ? a.T : 0);
    __nv_bfloat16 *xs = static_cast<__nv_bfloat16 *>(a.xperm);
    const int64_t n = rows * (a.H / 8);
    cudaError_t err = launch_k(k_gather_x, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
                               static_cast<const __nv_bfloat16 *>(a.x), a.T, a.H, a.sorted, A, a.k, rows, xs);
    if (err != cudaSuccess) return err;
    TcP p{};
    tc_common(p, a);
    p.rows = a.I;
    p.half_rows = 0;
    p.K = a.H;
    p.s[0] = a.gate.s;
    p.s[1] = a.up.s;
    p.s_stride[0] = a.gate.ss;
    p.s_stride[1] = a.up.ss;
    p.s_sh[0] = a.gate_sh.s;
    p.s_sh[1] = a.up_sh.s;
    p.b_sh_row0 = A;
    p.out = a.h;
    p.out_ld = a.h_ld;
    p.sh_out_row0 = a.sh_h_row0;
    p.hperm = static_cast<__nv_bfloat16 *>(a.hperm);
    p.gateup = 1;
    return tc_go(p, a.gate, a.up, a.gate_sh, a.up_sh, xs, rows, num_sms, st, a.E + 1);
}

cudaError_t launch_ffn_tc_down(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    if (!a.routed && !a.shared) return cudaSuccess;
    __nv_bfloat16 *hperm = static_cast<__nv_bfloat16 *>(a.hperm);
    const int64_t rows = std::max(a.routed ? (int64_t)a.T * a.k : (int64_t)0,
                                  a.shared ? a.sh_h_row0 + a.T : (int64_t)0);
    if (!a.hperm_ready) {       // h given in f32: round to bf16 and permute it here
        const int64_t n = rows * (a.I / 8);
        cudaError_t err = launch_k(k_perm_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
                                   (const float *)a.h, a.h_ld, rows, a.I, hperm);
        if (err != cudaSuccess) return err;
    }
    TcP p{};
    tc_common(p, a);
    p.rows = a.H;
    p.half_rows = TC_HALF;
    p.K = a.I;
    p.s[0] = p.s[1] = a.down.s;
    p.s_stride[0] = p.s_stride[1] = a.down.ss;
    p.s_sh[0] = p.s_sh[1] = a.down_sh.s;
    p.b_sh_row0 = a.sh_h_row0;
    p.out = a.y;
    p.out_ld = a.y_ld;
    p.sh_out_row0 = a.sh_y_row0;
    p.hperm = nullptr;
    p.gateup = 0;
    return tc_go(p, a.down, a.down, a.down_sh, a.down_sh, hperm, rows, num_sms, st, a.E + 1);
}

}  // namespace qrx
