// qrx_internal.h -- launchers shared between the qrx .cu files (not public).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qrx.h"

namespace qrx {

// Launches made while g_pdl is set carry the programmatic-stream-serialization
// attribute (the layer forward sets it for every kernel after its first).
extern thread_local bool g_pdl;

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = g_pdl ? attr : nullptr;
    cfg.numAttrs = g_pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// device status flag (one per device, in k_quant.cu)
cudaError_t read_and_clear_device_flag(int *flag);

cudaError_t launch_requant_fp8(const uint8_t *w8, int64_t rows, int64_t K, int64_t ld8, const float *bscale,
                              int wbits, uint8_t *q, int64_t ldq, float *scale, int64_t lds, cudaStream_t st);
cudaError_t launch_quantize_weights(const float *w, int64_t rows, int64_t K, int wbits,
                                    uint8_t *q, int64_t ldq, float *scale, int64_t lds,
                                    cudaStream_t st);
cudaError_t launch_quantize_act_q8(const float *x, int64_t nblocks, int8_t *xq, float *xd,
                                   cudaStream_t st);
cudaError_t launch_block_dots_q8(int wbits, const uint8_t *q, int64_t rows, int64_t K,
                                 const int8_t *xq, int32_t *acc, cudaStream_t st);

// router: partial dots then selection
struct RouterArgs {
    const void *x;          // f32 or bf16 [T][H]
    int x_bf16;
    const float *Wr;        // [E][H]
    const float *bias;      // [E]
    int T, H, E, G, Gk, k;
    float rsf;
    float *logits;          // [T][E] scratch
    int32_t *idx;           // [T][k]
    float *w;               // [T][k]
    double topp_thr;        // adaptive top-p: p * rsf; 0 = off
    uint32_t *zero;         // if set: zero[0, nzero) cleared by the logits kernel (scratch of the next kernels)
    int nzero;
    double *part;           // split-K scratch: slices x T x E doubles (null: no split kernel)
    int *tilecnt;           // split-K per-tile counters, zero between calls
};
// the logits kernel, then (select) the selection kernel
cudaError_t launch_router(const RouterArgs &a, cudaStream_t st, bool select = true);
// selection and permutation in one kernel, for small batches
bool select_permute_fused_ok(int T, int E, int G);
cudaError_t launch_select_permute(const RouterArgs &a, const qrx_perm &p, uint64_t *usage, cudaStream_t st);
cudaError_t launch_topp_prune(int32_t *idx, float *w, int T, int k, double thr, cudaStream_t st);

// usage (may be null): per-expert counters [E], += this call's counts
cudaError_t launch_permute(const int32_t *idx, int T, int k, int E, const qrx_perm &p,
                           cudaStream_t st, uint64_t *usage = nullptr);
cudaError_t launch_usage_add(const int32_t *counts, int E, uint64_t *usage, cudaStream_t st);

// One packed matrix of every expert: expert e's codes at q + e*sq bytes,
// its row scales at s + e*ss floats (qrx_mat).
struct MatRef {
    const uint8_t *q;
    const float *s;
    int64_t sq, ss;
};

// expert FFN over the union
struct FfnArgs {
    int wbits, afmt;
    int H, I, E, k, T;
    // routed experts (unused if !routed), shared expert (unused if !shared)
    MatRef gate, up, down;
    MatRef gate_sh, up_sh, down_sh;
    int routed, shared;
    const int32_t *offsets, *sorted, *union_ids, *n_union;
    // activations
    const void *x;          // f32 / bf16 [T][H]
    const int8_t *xq;       // Q8 [T][H]
    const float *xd;        // Q8 [T][H/32]
    unsigned char *xrec;    // scratch: gate/up input digit records [T][record bytes]
    int prep_records;       // launch_ffn_gateup first builds xrec from x / xq, xd
    unsigned char *hrec;    // scratch: down input digit records, one per h row
    void *xperm;            // scratch (tensor-core path): bf16 x, chunk-permuted [T][H]
    void *hperm;            // scratch (tensor-core path): bf16 h, chunk-permuted, one per h row
    int hperm_ready;        // the gate/up call of this layer already wrote hperm
    // positions: routed p in [0, T*k), shared p = T*k + t
    float *h;               // [P][I] intermediate (gate/up output, down input)
    float *y;               // [P][H]
    int64_t h_ld, y_ld;     // row strides (elements)
    // where the shared expert's rows live: h + sh_h_off*h_ld, y + sh_y_off*y_ld
    int64_t sh_h_row0, sh_y_row0;
};
cudaError_t launch_act_digits(const FfnArgs &a, cudaStream_t st);
bool ffn_use_tc(const FfnArgs &a);
bool tc_shape_ok(int afmt, int wbits, int64_t T, int64_t H, int64_t I);
cudaError_t launch_ffn_tc_gateup(const FfnArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_tc_down(const FfnArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_gateup(const FfnArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_ffn_down(const FfnArgs &a, int num_sms, cudaStream_t st);
// decode GEMV (T <= 4): whether it takes this call, and its launches
bool g2_use(const FfnArgs &a);
cudaError_t launch_g2_gateup(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe = nullptr);
cudaError_t launch_g2_down(const FfnArgs &a, int num_sms, cudaStream_t st, int32_t *probe = nullptr);
// Layer forward with the decode GEMV: the gate/up launch also makes the
// selection and the permutation from the router logits, and the down launch
// also applies the weighted combine.
struct G2Fuse {
    const float *logits, *bias;   // router logits [T][E], score-correction bias [E]
    int G, Gk;
    float rsf;
    double topp_thr;              // adaptive top-p threshold p * rsf (0: off)
    int32_t *idx;                 // [T][k] chosen experts (out)
    float *w;                     // [T][k] weights (out)
    uint64_t *usage;              // per-expert counters (may be null)
    int32_t *counts, *inv;        // permutation outputs besides those in FfnArgs
    int32_t *tab;                 // compact slot table: 4 + 4 * (min(E, T*k) + 1) ints
    int32_t *cnt;                 // combine counters: g2_down_groups() ints
    float *out;                   // [T][H] layer output (down launch; null: no combine)
    uint32_t *hmax;               // [T*k + T] largest |h| per h row (bits), zeroed by the logits kernel
};
bool g2_fuse_ok(const FfnArgs &a, int G, int Gk);
// multi-token GEMV on tensor cores (2 <= T <= 64, int4 / int8 weights)
bool gm_use(const FfnArgs &a);
cudaError_t launch_gm_gateup(const FfnArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_gm_down(const FfnArgs &a, int num_sms, cudaStream_t st);
int g2_down_groups(const FfnArgs &a);
cudaError_t launch_g2_gateup_fused(const FfnArgs &a, const G2Fuse &f, int num_sms, cudaStream_t st);
cudaError_t launch_g2_down_fused(const FfnArgs &a, const G2Fuse &f, int num_sms, cudaStream_t st);

cudaError_t launch_combine(const float *y_sorted, const float *y_sh, const float *w,
                           const int32_t *inv, int T, int k, int H, float *out,
                           cudaStream_t st);

}  // namespace qrx
