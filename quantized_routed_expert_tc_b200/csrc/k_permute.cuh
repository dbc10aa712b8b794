// k_permute.cuh -- batch-union permutation: a deterministic, stable counting
// sort of the T*k assignments a = t*k + j by expert.
//
// README "JustVugg/colibri", section "已实现的功能": batch-union MoE, each
// unique expert of a batch read once and applied to every position routed to
// it; blog "GLM-5.2 on slow computers", "让它变得可以忍受的那些装置": the same
// expert in a batch is read only once.
//
// A slot with expert -1 (dropped by adaptive top-p) takes no position: it is
// not counted and its inv entry is -1.  When a usage array is given, the
// per-expert counts of this call are added to it (expert-usage histogram).
//
// One CTA of 32 warps.  Warp w owns a contiguous segment of assignments.
// Pass 1 counts experts per segment (ballot-free: __match_any_sync leaders add
// their group's size), a column scan over warps turns the counts into each
// segment's first slot per expert, and pass 2 walks each segment again in the
// same order placing assignments -- so the order never depends on timing.
#pragma once
#include "qrx_dev.cuh"

namespace qrx {

constexpr int PERM_WARPS = 32;

__device__ __forceinline__ int block_exclusive_scan_1024(int v, int *tmp, int &total)
{
    // tmp: 32 ints of shared memory; blockDim.x == 1024
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) tmp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int w = tmp[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        tmp[lane] = wi - w;          // exclusive prefix of warp totals
        if (lane == 31) tmp[32] = wi;
    }
    __syncthreads();
    const int r = tmp[wid] + inc - v;
    total = tmp[32];
    __syncthreads();
    return r;
}

// The permutation by one CTA of 1024 threads; psm: (PERM_WARPS * E + 40) ints
// of shared memory.  Every thread of the CTA calls it.
__device__ __forceinline__ void permute_cta(const int32_t *__restrict__ idx, int A, int E, const qrx_perm &p,
                                            uint64_t *__restrict__ usage, int *psm)
{
    int *whist = psm;                          // [PERM_WARPS][E]
    int *tmp = psm + PERM_WARPS * E;           // [33]
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int i = tid; i < PERM_WARPS * E; i += 1024) whist[i] = 0;
    __syncthreads();

    const int seg = (A + PERM_WARPS - 1) / PERM_WARPS;
    const int a0 = min(A, wid * seg), a1 = min(A, a0 + seg);
    for (int base = a0; base < a1; base += 32) {
        const int a = base + lane;
        int e = -1;
        if (a < a1) {
            e = idx[a];
            // -1: a slot dropped by adaptive top-p; anything else outside [0, E) is an error
            if (e != -1 && (e < 0 || e >= E)) raise_status(DERR_BADIDX);
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) whist[wid * E + e] += __popc(peers);
    }
    __syncthreads();

    // per expert: total count and each segment's start within the expert
    int cnt = 0;
    if (tid < E) {
        for (int w = 0; w < PERM_WARPS; ++w) {
            const int c = whist[w * E + tid];
            whist[w * E + tid] = cnt;
            cnt += c;
        }
    }
    int total;
    const int off = block_exclusive_scan_1024(tid < E ? cnt : 0, tmp, total);
    const int present = (tid < E && cnt > 0) ? 1 : 0;
    int nu;
    const int upos = block_exclusive_scan_1024(present, tmp, nu);
    if (tid < E) {
        p.counts[tid] = cnt;
        p.offsets[tid] = off;
        if (usage && cnt) atomicAdd(reinterpret_cast<unsigned long long *>(usage + tid), (unsigned long long)cnt);
        if (present) p.union_ids[upos] = tid;
        for (int w = 0; w < PERM_WARPS; ++w) whist[w * E + tid] += off;
    }
    if (tid == 0) {
        p.offsets[E] = total;
        *p.n_union = nu;
    }
    __syncthreads();

    for (int base = a0; base < a1; base += 32) {
        const int a = base + lane;
        int e = -1;
        if (a < a1) {
            e = idx[a];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int pos = -1;
        if (e >= 0) pos = whist[wid * E + e] + rank;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) whist[wid * E + e] += __popc(peers);
        __syncwarp();
        if (a < a1) {
            p.inv[a] = pos;
            if (pos >= 0) p.sorted[pos] = a;
        }
    }
}

__global__ void __launch_bounds__(1024, 1) k_permute(const int32_t *__restrict__ idx, int A, int E,
                                                     qrx_perm p, uint64_t *__restrict__ usage)
{
    extern __shared__ __align__(16) int psm[];
    pdl_wait();
    pdl_trigger();
    permute_cta(idx, A, E, p, usage, psm);
}

__host__ __device__ inline size_t permute_smem_bytes(int E) { return ((size_t)PERM_WARPS * E + 40) * sizeof(int); }

cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, const qrx_perm &p,
                           cudaStream_t st, uint64_t *usage)
{
    const size_t smem = permute_smem_bytes(E);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
        if (err != cudaSuccess) return err;
    }
    return launch_k(k_permute, dim3(1), dim3(1024), smem, st, idx, T * k, E, p, usage);
}

// Expert-usage histogram (README "JustVugg/colibri", "快速开始": the engine
// records which experts a run routes to): usage[e] += counts[e].
__global__ void __launch_bounds__(256) k_usage_add(const int32_t *__restrict__ counts, int E,
                                                   uint64_t *__restrict__ usage)
{
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < E && counts[e] > 0)
        atomicAdd(reinterpret_cast<unsigned long long *>(usage + e), (unsigned long long)counts[e]);
}

cudaError_t launch_usage_add(const int32_t *counts, int E, uint64_t *usage, cudaStream_t st)
{
    return launch_k(k_usage_add, dim3((unsigned)((E + 255) / 256)), dim3(256), 0, st, counts, E, usage);
}

}  // namespace qrx
