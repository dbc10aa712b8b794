// k_ffn_tc.cuh -- expert FFN over the batch union as grouped GEMMs on the
// tcgen05 tensor cores, for batches with many tokens per expert (prefill,
// long verify batches) and bf16 activations.
//
// README "JustVugg/colibri", section "已实现的功能": batch-union MoE (each
// unique expert of a batch is read once and applied to all positions routed
// to it); packed int4 weights with per-row scales, dequantised on use.  With
// ~64 tokens per expert the work is a dense contraction, so it runs on the
// tensor cores: int4 codes are exact in bf16, products accumulate in f32, and
// the per-row scale multiplies the accumulator in the epilogue.
//
// Tiles.  A work item is (slot, 128 weight rows, up to 256 tokens): the
// weights are the MMA's M side and the tokens its N side, K advances in
// stages of 64 (one 128-byte swizzle atom of bf16).  Roles per CTA (one CTA
// per SM, persistent over items):
//   warps 0-3  loaders: cp.async of the int4 weight rows (each thread owns one
//              row) and of the token rows; each thread dequantises its own
//              row into the 128B-swizzled K-major A tile, then arrives on the
//              stage's "full" mbarrier;
//   warp 4     allocates 512 TMEM columns (two 128x256 f32 accumulators) and
//              issues tcgen05.mma (M=128, N<=256, K=16, four per stage); each
//              stage is released with tcgen05.commit to its "empty" mbarrier,
//              each finished item with a commit to its accumulator's "full";
//   warps 5-8  epilogue: tcgen05.ld of the accumulator, row scales, SwiGLU
//              (gate/up) or the output rows (down), stores.
// Dequantisation writes the 8 codes of a packed word in the order
// (0,4,1,5,2,6,3,7); the token rows (and h for the down projection) are kept
// in the same order within every 8-element chunk, so the contraction is
// unchanged.  All mbarrier waits are bounded; a timeout raises the device
// status flag and every role leaves its loops before TMEM is freed.
#pragma once
#include "qrx_dev.cuh"

namespace qrx {

constexpr int TC_M = 128, TC_BK = 64, TC_NMAX = 256, TC_STAGES = 4, TC_LOOKAHEAD = 3;
constexpr int TC_LOADERS = 128, TC_THREADS = 288;                // 9 warps
constexpr int TC_A_BYTES = TC_M * 128;                           // bf16 A tile, 16 KB
constexpr int TC_RAW_BYTES = TC_M * 32;                          // int4 A tile, 4 KB
constexpr int TC_B_BYTES = TC_NMAX * 128;                        // bf16 B tile, 32 KB
constexpr int TC_STAGE_BYTES = TC_A_BYTES + TC_B_BYTES + TC_RAW_BYTES;
// dynamic shared memory: 1024-byte alignment slack, the stages, 128 bytes of
// barriers and flags, the item prefix over up to maxslots slots
__host__ __device__ constexpr int tc_smem_bytes(int maxslots)
{
    return 1024 + TC_STAGE_BYTES * TC_STAGES + 128 + (maxslots + 2) * 8;
}

// Position p within an 8-element chunk holds element kPermTC[p].
__host__ __device__ constexpr int tc_perm(int p) { return (p & 1) ? 4 + (p >> 1) : (p >> 1); }
__host__ __device__ constexpr int tc_inv_perm(int e) { return e < 4 ? 2 * e : 2 * (e - 4) + 1; }

struct TcP {
    int rows, K, row_bytes, mtiles, kstages;
    const uint8_t *w;       // routed weights, expert stride w_stride bytes
    int64_t w_stride;
    const float *s;         // routed row scales, expert stride s_stride
    int64_t s_stride;
    const uint8_t *w_sh;
    const float *s_sh;
    int routed, shared, E, k, T;
    const int32_t *offsets, *sorted, *union_ids, *n_union;
    const __nv_bfloat16 *bsrc;   // B rows (bf16, chunk-permuted): tokens (gate/up) or h rows (down)
    int64_t sh_in_row0;          // down: B row of the shared expert's first token
    float *out;                  // gate/up: h f32 [rows of positions][I]; down: y f32
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
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// Item geometry for slot s: token tiles of at most 256, balanced, multiple of 16.
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

__global__ void __launch_bounds__(TC_THREADS, 1) k_ffn_tc(const TcP p)
{
    extern __shared__ __align__(1024) unsigned char tsm_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *tsm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *ctl = tsm + TC_STAGE_BYTES * TC_STAGES;
    uint64_t *full = reinterpret_cast<uint64_t *>(ctl);            // [STAGES]
    uint64_t *empty = full + TC_STAGES;                            // [STAGES]
    uint64_t *acc_full = empty + TC_STAGES;                        // [2]
    uint64_t *acc_empty = acc_full + 2;                            // [2]
    uint64_t *drain = acc_empty + 2;                               // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int64_t *pre = reinterpret_cast<int64_t *>(ctl + 128);        // [nslots + 1] item prefix

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    const int nu = p.routed ? *p.n_union : 0;
    const int nslots = nu + (p.shared ? 1 : 0);

    if (tid == 0) {
        for (int i = 0; i < TC_STAGES; ++i) {
            mbar_init(smem_u32(&full[i]), TC_LOADERS);
            mbar_init(smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 4);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // item prefix over slots (warp 5): items of slot s = ntiles * mtiles
    if (warp == 5) {
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

    // decode item -> (slot, m tile, token tile)
    auto decode = [&](int64_t it, int &s, int &mt, int &n0, int &nv, int &nn) {
        int lo = 0, hi = nslots;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= it) lo = mid; else hi = mid;
        }
        s = lo;
        const TcSlot sl = tc_slot(p, s, nu);
        const int64_t r = it - pre[s];
        const int ni = (int)(r / p.mtiles);
        mt = (int)(r % p.mtiles);
        n0 = ni * sl.nbase;
        nv = min(sl.nbase, sl.ntok - n0);
        nn = sl.nbase;
    };

    if (warp < 4) {
        // ================= loaders =================
        const int row = tid;                       // weight row within the tile
        int64_t g = 0;                             // global stage counter
        int64_t issued = 0;
        // per-item state for the stages being issued
        for (int64_t it = blockIdx.x; it < nitems && !*abort_flag; it += gridDim.x) {
            int s, mt, n0, nv, nn;
            decode(it, s, mt, n0, nv, nn);
            const bool routed = s < nu;
            int e = 0, p0 = 0;
            if (routed) {
                e = p.union_ids[s];
                e = (e >= 0 && e < p.E) ? e : 0;
                p0 = p.offsets[e];
            }
            const uint8_t *W = (routed ? p.w + (int64_t)e * p.w_stride : p.w_sh) +
                               ((int64_t)mt * TC_M + row) * p.row_bytes;
            // B source row of token n of this item
            auto brow = [&](int n) -> int64_t {
                const int i = n0 + n;
                if (p.gateup) return routed ? p.sorted[p0 + i] / p.k : i;
                return routed ? p0 + i : p.sh_in_row0 + i;
            };
            auto issue_stage = [&](int kb, int64_t gs) {
                const int st = (int)(gs % TC_STAGES);
                unsigned char *sb = tsm + (size_t)st * TC_STAGE_BYTES;
                // wait until the MMA has released this stage
                if (*abort_flag) return;
                if (gs >= TC_STAGES &&
                    !mbar_wait(smem_u32(&empty[st]), (uint32_t)(((gs / TC_STAGES) - 1) & 1))) {
                    *abort_flag = 1;
                    raise_status(DERR_TIMEOUT);
                    return;
                }
                const uint32_t raw = smem_u32(sb + TC_A_BYTES + TC_B_BYTES) + row * 32;
                cp_async16(raw, W + kb * 32, 16);
                cp_async16(raw + 16, W + kb * 32 + 16, 16);
                const uint32_t bt = smem_u32(sb + TC_A_BYTES);
                for (int q = tid; q < nn * 8; q += TC_LOADERS) {
                    const int n = q >> 3, c = q & 7;
                    const bool ok = n < nv;
                    const __nv_bfloat16 *src = p.bsrc + (ok ? brow(n) : 0) * (int64_t)p.K + kb * 64 + c * 8;
                    cp_async16(bt + n * 128 + ((c ^ (n & 7)) << 4), src, ok ? 16 : 0);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            };
            // prologue: the first stages of this item
            int kissue = 0;
            for (; kissue < TC_LOOKAHEAD && kissue < p.kstages; ++kissue) issue_stage(kissue, issued++);
            for (int kb = 0; kb < p.kstages && !*abort_flag; ++kb, ++g) {
                if (kissue < p.kstages) {
                    issue_stage(kissue++, issued++);
                } else {
                    asm volatile("cp.async.commit_group;" ::: "memory");
                }
                asm volatile("cp.async.wait_group %0;" ::"n"(TC_LOOKAHEAD) : "memory");
                const int st = (int)(g % TC_STAGES);
                unsigned char *sb = tsm + (size_t)st * TC_STAGE_BYTES;
                // dequantise this thread's row: 64 codes -> 8 swizzled 16-byte chunks
                const uint4 *rawp = reinterpret_cast<const uint4 *>(sb + TC_A_BYTES + TC_B_BYTES + row * 32);
                const uint4 r0 = rawp[0], r1 = rawp[1];
                const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t o = words[j] ^ 0x88888888u;
                    uint32_t q[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t v = ((o >> (4 * h)) & 0x000F000Fu) | 0x43004300u;
                        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v);
                        b = __hsub2(b, off);
                        q[h] = *reinterpret_cast<uint32_t *>(&b);
                    }
                    *reinterpret_cast<uint4 *>(sb + row * 128 + ((j ^ (row & 7)) << 4)) =
                        make_uint4(q[0], q[1], q[2], q[3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(smem_u32(&full[st]));
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 4) {
        // ================= MMA issue =================
        int64_t g = 0;
        int local = 0;
        for (int64_t it = blockIdx.x; it < nitems && !*abort_flag; it += gridDim.x, ++local) {
            int s, mt, n0, nv, nn;
            decode(it, s, mt, n0, nv, nn);
            const int a = local & 1;
            if (local >= 2 &&
                !mbar_wait(smem_u32(&acc_empty[a]), (uint32_t)(((local >> 1) - 1) & 1))) {
                *abort_flag = 1;
                raise_status(DERR_TIMEOUT);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t d = tmem + (uint32_t)(a * TC_NMAX);
            const uint32_t idesc = tc_idesc(nn);
            for (int kb = 0; kb < p.kstages; ++kb, ++g) {
                const int st = (int)(g % TC_STAGES);
                if (!mbar_wait(smem_u32(&full[st]), (uint32_t)((g / TC_STAGES) & 1))) {
                    *abort_flag = 1;
                    raise_status(DERR_TIMEOUT);
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (lane == 0) {
                    unsigned char *sb = tsm + (size_t)st * TC_STAGE_BYTES;
                    const uint64_t da = tc_desc_sw128(smem_u32(sb));
                    const uint64_t db = tc_desc_sw128(smem_u32(sb + TC_A_BYTES));
#pragma unroll
                    for (int k = 0; k < TC_BK / 16; ++k) {
                        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred pd;\n\t"
                            "setp.ne.b32 pd, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, pd;\n\t}"
                            ::"r"(d), "l"(da + 2 * k), "l"(db + 2 * k), "r"(idesc), "r"(acc),
                            "r"(0), "r"(0), "r"(0), "r"(0)
                            : "memory");
                    }
                    asm volatile(
                        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                            smem_u32(&empty[st]))
                        : "memory");
                }
                __syncwarp();
            }
            if (*abort_flag) break;
            if (lane == 0)
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                        smem_u32(&acc_full[a]))
                    : "memory");
            __syncwarp();
        }
        // every MMA issued above has completed before TMEM is freed
        if (lane == 0) {
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    smem_u32(drain))
                : "memory");
            if (!mbar_wait(smem_u32(drain), 0u)) raise_status(DERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ================= epilogue (warps 5..8) =================
        const int q4 = warp & 3;                   // TMEM lane quarter of this warp
        const int lrow = q4 * 32 + lane;           // accumulator row = weight row in tile
        int local = 0;
        for (int64_t it = blockIdx.x; it < nitems && !*abort_flag; it += gridDim.x, ++local) {
            int s, mt, n0, nv, nn;
            decode(it, s, mt, n0, nv, nn);
            const bool routed = s < nu;
            int e = 0, p0 = 0;
            if (routed) {
                e = p.union_ids[s];
                e = (e >= 0 && e < p.E) ? e : 0;
                p0 = p.offsets[e];
            }
            const int rowg = mt * TC_M + lrow;
            const float sc = (routed ? p.s + (int64_t)e * p.s_stride : p.s_sh)[rowg];
            const int a = local & 1;
            if (!mbar_wait(smem_u32(&acc_full[a]), (uint32_t)((local >> 1) & 1))) {
                *abort_flag = 1;
                raise_status(DERR_TIMEOUT);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            for (int c0 = 0; c0 < nn; c0 += 16) {
                uint32_t v[16];
                const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(a * TC_NMAX + c0);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                      "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                      "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    const float acc = sc * __uint_as_float(v[j]);
                    const int i = n0 + n;
                    int orow;
                    if (p.gateup) {
                        const float other = __shfl_xor_sync(0xffffffffu, acc, 1);
                        if ((lane & 1) || n >= nv) continue;
                        orow = routed ? p0 + i : (int)p.sh_out_row0 + i;
                        const int pair = rowg >> 1;
                        const float h = silu_mul(acc, other);
                        p.out[(int64_t)orow * p.out_ld + pair] = h;
                        if (p.hperm)
                            p.hperm[(int64_t)orow * (p.rows / 2) + (pair & ~7) + tc_inv_perm(pair & 7)] =
                                __float2bfloat16_rn(h);
                    } else {
                        if (n >= nv) continue;
                        orow = routed ? p0 + i : (int)p.sh_out_row0 + i;
                        p.out[(int64_t)orow * p.out_ld + rowg] = acc;
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 4) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// x (bf16 [T][K]) -> chunk-permuted copy; h (f32 rows, stride ld) -> bf16 chunk-permuted.
__global__ void __launch_bounds__(256) k_perm_bf16(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                   int K, __nv_bfloat16 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= rows * (K / 8)) return;
    const uint4 v = reinterpret_cast<const uint4 *>(x)[id];
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&v);
    __nv_bfloat16 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = e[tc_perm(q)];
    reinterpret_cast<uint4 *>(out)[id] = *reinterpret_cast<const uint4 *>(o);
}

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

constexpr int TC_MIN_T = 256;   // tokens from which the tensor-core path is used

bool ffn_use_tc(const FfnArgs &a)
{
    return a.afmt == QRX_A_BF16 && a.wbits == 4 && a.T >= TC_MIN_T && (2 * a.I) % TC_M == 0 &&
           a.H % TC_M == 0 && a.H % TC_BK == 0 && a.I % TC_BK == 0 && a.xperm && a.hperm;
}

static cudaError_t tc_go(TcP &p, int num_sms, cudaStream_t st, int maxslots)
{
    p.row_bytes = p.K / 2;
    p.mtiles = p.rows / TC_M;
    p.kstages = p.K / TC_BK;
    const int smem = tc_smem_bytes(maxslots);
    static unsigned long long configured = 0;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || !(configured >> dev & 1ull)) {
        err = cudaFuncSetAttribute(k_ffn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM_MAX);
        if (err != cudaSuccess) return err;
        if (dev < 64) configured |= 1ull << dev;
    }
    if (smem > GV_SMEM_MAX) return cudaErrorInvalidValue;
    return launch_k(k_ffn_tc, dim3(num_sms), dim3(TC_THREADS), (size_t)smem, st, p);
}

static void tc_common(TcP &p, const FfnArgs &a)
{
    p.routed = a.routed;
    p.shared = a.shared;
    p.E = a.E;
    p.k = a.k;
    p.T = a.T;
    p.offsets = a.offsets;
    p.sorted = a.sorted;
    p.union_ids = a.union_ids;
    p.n_union = a.n_union;
}

cudaError_t launch_ffn_tc_gateup(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    __nv_bfloat16 *xperm = static_cast<__nv_bfloat16 *>(a.xperm);
    const int64_t n = (int64_t)a.T * (a.H / 8);
    cudaError_t err = launch_k(k_perm_bf16, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
                               static_cast<const __nv_bfloat16 *>(a.x), (int64_t)a.T, a.H, xperm);
    if (err != cudaSuccess) return err;
    TcP p{};
    tc_common(p, a);
    p.rows = 2 * a.I;
    p.K = a.H;
    p.w = a.w13;
    p.w_stride = (int64_t)2 * a.I * (a.H / 2);
    p.s = a.s13;
    p.s_stride = 2 * a.I;
    p.w_sh = a.w13_sh;
    p.s_sh = a.s13_sh;
    p.bsrc = xperm;
    p.sh_in_row0 = 0;
    p.out = a.h;
    p.out_ld = a.h_ld;
    p.sh_out_row0 = a.sh_h_row0;
    p.hperm = static_cast<__nv_bfloat16 *>(a.hperm);
    p.gateup = 1;
    return tc_go(p, num_sms, st, a.E + 1);
}

cudaError_t launch_ffn_tc_down(const FfnArgs &a, int num_sms, cudaStream_t st)
{
    __nv_bfloat16 *hperm = static_cast<__nv_bfloat16 *>(a.hperm);
    if (!a.hperm_ready) {       // h given in f32: round to bf16 and permute it here
        const int64_t rows = max(a.routed ? (int64_t)a.T * a.k : 0, a.shared ? a.sh_h_row0 + a.T : 0);
        const int64_t n = rows * (a.I / 8);
        cudaError_t err = launch_k(k_perm_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st,
                                   (const float *)a.h, a.h_ld, rows, a.I, hperm);
        if (err != cudaSuccess) return err;
    }
    TcP p{};
    tc_common(p, a);
    p.rows = a.H;
    p.K = a.I;
    p.w = a.w2;
    p.w_stride = (int64_t)a.H * (a.I / 2);
    p.s = a.s2;
    p.s_stride = a.H;
    p.w_sh = a.w2_sh;
    p.s_sh = a.s2_sh;
    p.bsrc = hperm;
    p.sh_in_row0 = a.sh_h_row0;
    p.out = a.y;
    p.out_ld = a.y_ld;
    p.sh_out_row0 = a.sh_y_row0;
    p.hperm = nullptr;
    p.gateup = 0;
    return tc_go(p, num_sms, st, a.E + 1);
}

}  // namespace qrx
