/*
 * qrx.h -- C ABI of libqrx: the routed-MoE layer forward over packed low-bit
 * expert weights, on one NVIDIA B200 (sm_100a).
 *
 * The operation is the MoE layer of GLM-5.2 as the colibri pages describe it:
 *   - colibri README ("JustVugg/colibri"), section "已实现的功能" (implemented
 *     features): DeepSeek-V3-like sigmoid router (noaux_tc,
 *     routed_scaling_factor), a shared expert, Q8_0-style int8-activation
 *     integer dot kernels, int8 / packed int4 / packed int2 weights with
 *     per-row scales dequantised on use, and the batch-union MoE (each unique
 *     expert of a batch read once, applied to every position routed to it);
 *   - blog "GLM-5.2 on slow computers", section "让它变得可以忍受的那些装置":
 *     the same expert in a batch is read only once; int4 container with
 *     per-row scale, dequant-on-use;
 *   - README sections "快速开始" and "如何测试，按顺序": adaptive expert top-p
 *     (--topp) and the per-expert usage record; "已实现的功能": the FP8
 *     (128x128 block scales) -> int4 converter.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller (for
 *     example torch tensors' data_ptr()), except where a call says "host".
 *     The library never frees or keeps them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream and never synchronise
 *     the host, except qrx_last_error, qrx_moe_forward_hostio and the
 *     query functions.
 *   - Argument checks are synchronous and happen before any launch; a
 *     failing check returns a negative QRX_E* code and launches nothing.
 *   - Kernels that detect a bad value at run time (an expert index out of
 *     range, an exhausted bounded wait) set a sticky device flag;
 *     qrx_last_error() synchronises the device and reports it.
 *   - libqrx_check.so, the same library built with -DQRX_CHECK, has this
 *     ABI and these results; its kernels also test every index they take
 *     from data (permutation positions, token rows, inv entries) against the
 *     buffer it addresses, skip a miss and report it as QRX_EDEVICE.
 *   - Calls are not thread-safe with respect to the same workspace.
 *
 * Tensor layouts (row-major, C order):
 *   x        [T][H]      f32 (QRX_A_F32, QRX_A_Q8_0) or bf16 (QRX_A_BF16)
 *   W_router [E][H]      f32;  bias [E] f32 (score-correction bias)
 *   topk_idx [T][k]      int32 (-1: a slot dropped by adaptive top-p);
 *   topk_w   [T][k]      f32 (0 for a dropped slot)
 *   Expert weights (qrx_experts): three packed matrices per expert in the
 *   [out][in] orientation, each with per-row f32 scales, in the container the
 *   README and the blog describe (int4 container with a per-row scale,
 *   dequantised on use) and read in place, never repacked:
 *     gate [I][H*b/8] uint8, scales [I]
 *     up   [I][H*b/8] uint8, scales [I]
 *     down [H][I*b/8] uint8, scales [H]
 *   Expert e's matrix starts expert_stride_q bytes after expert e-1's, its
 *   scales expert_stride_s floats after (n = E routed experts, or 1 shared);
 *   rows are contiguous (K*b/8 bytes each).
 *   (b = 8, 4 or 2 bits; packed fields as in the README: int4 low nibble
 *   first, int2 lowest bit pair first, two's-complement codes.)
 *   Assignment a = t*k + j.  Sorted order groups assignments by expert,
 *   stable in a; position p indexes that order; h and y rows are positions.
 */
#ifndef QRX_H
#define QRX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define QRX_OK 0
#define QRX_EINVAL (-1)        /* NULL pointer, bad size, T <= 0, ... */
#define QRX_EUNSUPPORTED (-2)  /* configuration outside what the kernels handle */
#define QRX_ECUDA (-3)         /* a CUDA runtime call failed */
#define QRX_ETIMEOUT (-4)      /* a bounded device wait gave up */
#define QRX_EDEVICE (-5)       /* a kernel saw an invalid value (sticky flag) */
#define QRX_ENOSPACE (-6)      /* workspace smaller than qrx_workspace_bytes */

typedef enum { QRX_W_INT8 = 8, QRX_W_INT4 = 4, QRX_W_INT2 = 2 } qrx_wfmt;
typedef enum { QRX_A_F32 = 0, QRX_A_Q8_0 = 1, QRX_A_BF16 = 2 } qrx_afmt;

/* Layer configuration (the README's router knobs plus sizes and formats). */
typedef struct {
    int32_t hidden;                /* H */
    int32_t n_experts;             /* E routed experts */
    int32_t inter;                 /* I expert intermediate size */
    int32_t n_group;               /* G expert groups (contiguous, E/G each) */
    int32_t topk_group;            /* Gk groups kept per token */
    int32_t top_k;                 /* k experts per token */
    float routed_scaling_factor;   /* rsf */
    int32_t wfmt;                  /* qrx_wfmt of routed and shared experts */
    int32_t afmt;                  /* qrx_afmt of the activations */
} qrx_cfg;

/* One packed matrix of every expert (see layout above).  q and scale are
 * device pointers, 16-byte aligned; expert_stride_q is a multiple of 16
 * bytes and expert_stride_s a multiple of 4 floats (QRX_EINVAL otherwise).
 * A set of one expert (the shared expert) ignores both strides. */
typedef struct {
    const uint8_t *q;          /* codes of expert 0: [rows][K*b/8] */
    const float *scale;        /* row scales of expert 0: [rows] */
    int64_t expert_stride_q;   /* bytes from one expert's codes to the next */
    int64_t expert_stride_s;   /* floats from one expert's scales to the next */
} qrx_mat;

/* An expert set: the SwiGLU FFN's three matrices (README "已实现的功能":
 * SwiGLU experts with per-row scales; blog "让它变得可以忍受的那些装置": int4
 * container with per-row scale, dequant-on-use). */
typedef struct {
    qrx_mat gate;   /* [I][H*b/8], scales [I] */
    qrx_mat up;     /* [I][H*b/8], scales [I] */
    qrx_mat down;   /* [H][I*b/8], scales [H] */
} qrx_experts;

/* Batch-union permutation buffers (device, int32):
 *   counts[E], offsets[E+1], sorted[T*k] (value a), inv[T*k] (value p),
 *   union_ids[E] (first *n_union valid, ascending), n_union[1]. */
typedef struct {
    int32_t *counts;
    int32_t *offsets;
    int32_t *sorted;
    int32_t *inv;
    int32_t *union_ids;
    int32_t *n_union;
} qrx_perm;

/* Activations handed to the expert FFN.
 *   QRX_A_F32:  x = f32 [T][H];        xq, xd unused.
 *   QRX_A_BF16: x = bf16 [T][H];       xq, xd unused.
 *   QRX_A_Q8_0: xq = int8 [T][H] and xd = f32 [T][H/32] from
 *               qrx_quantize_act_q8;   x unused.
 * Device pointers, 16-byte aligned (QRX_EINVAL otherwise). */
typedef struct {
    const void *x;
    const int8_t *xq;
    const float *xd;
} qrx_act;

/* ---- queries (host only, synchronous) ---------------------------------- */

/* Check a configuration (README "JustVugg/colibri", section "已实现的功能": a
 * DeepSeek-V3-like router over n_group groups keeping topk_group, top_k
 * experts, routed_scaling_factor; int8 / packed int4 / packed int2 experts;
 * f32 or Q8_0-style int8 activations).  QRX_EINVAL for non-positive sizes or a bad enum;
 * QRX_EUNSUPPORTED when: E % G != 0, Gk > G, Gk*E/G < k, k > 32, E > 1024,
 * H or I not a multiple of 64, or a row of H or I codes is not a supported
 * number of 16-byte chunks (1, 2, 4, 8, 16, 32, 64, 96, 128, 192 or 384). */
int qrx_validate(const qrx_cfg *cfg);

/* Bytes of scratch the calls below need for T tokens (a multiple of 256). */
size_t qrx_workspace_bytes(const qrx_cfg *cfg, int32_t T);

/* Which engine runs the expert FFN (gate/up + SwiGLU and down) of a call with
 * this configuration and T tokens (the routed, shared and whole-layer entry
 * points that take a workspace; README "JustVugg/colibri", section "已实现的功能":
 * the kernel for a shape is chosen by measurement):
 *   QRX_ENGINE_GEMV  the HBM-streaming integer GEMVs (any format): the
 *                    one-token decode GEMV, the multi-token GEMV with its dot
 *                    products on mma.sync tensor cores (2..64 tokens, int4 /
 *                    int8, or int2 with f32 / bf16 activations), or the dp4a
 *                    engine;
 *   QRX_ENGINE_TC    grouped GEMMs on the tcgen05 tensor cores: bf16
 *                    activations, int4 weights, T >= 256, H and I multiples
 *                    of 256, and a CUDA driver that provides tensor-map
 *                    encoding (without one, every shape reports the GEMV).
 * Returns QRX_EINVAL for an invalid configuration or T <= 0.  The
 * allocation-free entry point always uses the GEMV. */
#define QRX_ENGINE_GEMV 0
#define QRX_ENGINE_TC 1
int qrx_ffn_engine(const qrx_cfg *cfg, int32_t T);

/* Sticky device status: synchronises the current device, returns QRX_OK,
 * QRX_EDEVICE or QRX_ETIMEOUT (and clears the flag), or QRX_ECUDA if the
 * context reported an error. */
int qrx_last_error(void);
const char *qrx_strerror(int code);

/* ---- quantisation ------------------------------------------------------ */

/* Per-row symmetric quantisation of f32 rows into packed codes
 * (README "已实现的功能": per-row scale; tiny-layer workload: scale =
 * absmax/7 for int4, codes in [-8, 7], two per byte low nibble first).
 * scale_r = absmax_r / qmax (qmax = 127, 7, 1 for 8, 4, 2 bits), one f32
 * division; code = clamp(round-half-away(w / scale_r), qmin, qmax); a zero
 * row gets scale 0 and codes 0.
 *   w      [rows][K] f32 (device)
 *   q      output: row r at q + r*ldq bytes, K*wbits/8 bytes per row
 *   scale  output: scale of row r at scale[r*lds]
 * K must be a multiple of 32.  Bit-exact with the CPU reference. */
int qrx_quantize_weights(const float *w, int64_t rows, int64_t K, int32_t wbits,
                         uint8_t *q, int64_t ldq, float *scale, int64_t lds, void *stream);

/* FP8 checkpoint rows -> the same packed per-row container (README
 * "JustVugg/colibri", section "已实现的功能": the FP8->int4 converter
 * dequantises with 128x128 block scales and requantises for the engine).
 * Each value is f32(e4m3 code) * bscale[r/128][c/128] (one f32 multiply; a NaN
 * code counts as 0), then quantised as qrx_quantize_weights does.
 *   w8      [rows][K] FP8 e4m3 codes (device), row r at w8 + r*ld8 bytes
 *   bscale  [ceil(rows/128)][ceil(K/128)] f32 block scales (device, row-major)
 *   q, ldq, scale, lds: outputs as in qrx_quantize_weights
 * K must be a multiple of 32, ld8 a multiple of 4, w8 4-byte aligned.
 * Bit-exact with the CPU reference. */
int qrx_requant_fp8(const uint8_t *w8, int64_t rows, int64_t K, int64_t ld8, const float *bscale,
                    int32_t wbits, uint8_t *q, int64_t ldq, float *scale, int64_t lds, void *stream);

/* Q8_0-style activations (README "已实现的功能": integer dot with Q8_0-style
 * int8 activations; blocks of 32 with an f32 absmax scale):
 * d = amax/127, q = clamp(round-half-away(x * (127/amax)), -127, 127), a zero
 * block gives d = 0, q = 0.  x [T][H] f32 -> xq [T][H] int8, xd [T][H/32] f32.
 * H must be a multiple of 32.  Bit-exact with the CPU reference. */
int qrx_quantize_act_q8(const float *x, int64_t T, int64_t H, int8_t *xq, float *xd,
                        void *stream);

/* Exact int32 block accumulators acc[r][b] = sum over the 32-element block b
 * of code(r, i) * xq[i], through the same unpack and dp4a path as the FFN
 * kernels (the integer part of a Q8_0 dot; compared bit for bit in tests).
 *   q [rows][K*wbits/8], xq [K] int8, acc [rows][K/32] int32. */
int qrx_block_dots_q8(int32_t wbits, const uint8_t *q, int64_t rows, int64_t K,
                      const int8_t *xq, int32_t *acc, void *stream);

/* ---- the layer, step by step ------------------------------------------ */

/* Router (README "已实现的功能": DeepSeek-V3-like sigmoid router, noaux_tc,
 * routed_scaling_factor): logit = x . W_router[e] (f64 accumulation, rounded
 * to f32), s = sigmoid(logit), sc = s + bias (selection only); groups of E/G
 * contiguous experts scored by the sum of their two largest sc; the Gk best
 * groups kept (ties to the lower group); the k largest sc among their
 * experts (ties to the lower id) in descending order; weights
 * w_j = s_j / sum(s) * rsf.  x per cfg->afmt (f32 for F32 and Q8_0, bf16 for
 * BF16).  ws: at least qrx_workspace_bytes(cfg, T) bytes. */
int qrx_route(const qrx_cfg *cfg, const void *x, int32_t T, const float *W_router,
              const float *bias, int32_t *topk_idx, float *topk_w, void *ws,
              size_t ws_bytes, void *stream);

/* Batch-union permutation (README "已实现的功能": batch-union MoE; blog:
 * same expert read once per batch): a stable counting sort of the T*k
 * assignments by expert.  Deterministic.  An index of -1 marks a slot dropped
 * by adaptive top-p: it is not counted and its inv entry is -1.  Sets the
 * device error flag if an index is outside [0, E) and not -1. */
int qrx_permute(const qrx_cfg *cfg, const int32_t *topk_idx, int32_t T,
                const qrx_perm *perm, void *stream);

/* Adaptive expert top-p (README "JustVugg/colibri", section "快速开始": the
 * --topp knob, default 0.7; "社区基准（实测）": its measured effect), applied
 * in place to a router output topk_idx / topk_w [T][k] (device):
 * per token, slots are taken by weight, largest first (equal weights: the
 * lower slot first), their weights summed in double in that order, until the
 * sum reaches (double)p * (double)rsf; the other slots become idx = -1,
 * w = 0.  Kept weights are not renormalised.  p outside (0, 1) leaves the
 * arrays unchanged.  QRX_EINVAL for NULL arrays or a NaN p. */
int qrx_topp_prune(const qrx_cfg *cfg, int32_t *topk_idx, float *topk_w, int32_t T, float p,
                   void *stream);

/* Expert-usage histogram (README "JustVugg/colibri", "快速开始": the engine
 * records which experts a run routes to; "如何测试，按顺序": the STATS file):
 * usage[e] += perm->counts[e] for every expert, on device.  usage: caller-owned
 * device array of E uint64 counters, 8-byte aligned, set to zero by the caller
 * before the first call; calls on one stream accumulate in order. */
int qrx_usage_accumulate(const qrx_cfg *cfg, const qrx_perm *perm, uint64_t *usage, void *stream);

/* Routed experts' SwiGLU FFN over the batch union (README "JustVugg/colibri",
 * section "已实现的功能": batch-union MoE, int8 / packed int4 / packed int2
 * dequantised on use; blog "GLM-5.2 on slow computers", section
 * "让它变得可以忍受的那些装置": an expert shared by a batch is read once): for
 * each expert of the union, its gate/up rows are read once for all of its positions:
 * h = silu(s_g (Q_g x)) * (s_u (Q_u x)), then y = s_d (Q_d h') where h' is h
 * (F32), h rounded to bf16 (BF16) or h re-quantised to Q8_0 (Q8_0).
 *   h_sorted: [T*k][I] f32 output (may be NULL: workspace is used)
 *   y_sorted: [T*k][H] f32 output, rows in sorted order. */
int qrx_expert_ffn(const qrx_cfg *cfg, const qrx_experts *routed, const qrx_perm *perm,
                   const qrx_act *act, int32_t T, float *h_sorted, float *y_sorted,
                   void *ws, size_t ws_bytes, void *stream);

/* Down projection alone (the second half of the expert FFN above, README
 * "JustVugg/colibri", section "已实现的功能"), from a given h_sorted [T*k][I]
 * f32 (stage isolation: lets a test feed the reference's h). */
int qrx_expert_down(const qrx_cfg *cfg, const qrx_experts *routed, const qrx_perm *perm,
                    const float *h_sorted, int32_t T, float *y_sorted, void *ws,
                    size_t ws_bytes, void *stream);

/* The exact int32 accumulators of the Q8_0 path, for checking them bit for
 * bit (README "已实现的功能": Q8_0-style int8-activation integer dot kernels;
 * blocks of 32 codes with one f32 scale each).  These run the routed FFN's own
 * decode kernels (calls of T <= 4 tokens, cfg->afmt == QRX_A_Q8_0; otherwise
 * QRX_EUNSUPPORTED) with one more store: every 32-block's accumulator
 * acc_b = sum of code(row, i) * q8(act)[i] over the block, exactly as the
 * kernel forms it before scaling it by the block's d_b.
 *   qrx_expert_gateup_q8_sums: the gate/up stage of qrx_expert_ffn on act;
 *     h_sorted [T*k][I] f32 output; acc [T*k][2][I][H/32] int32 (gate rows,
 *     then up rows) for every routed position.
 *   qrx_expert_down_q8_sums: the down stage of qrx_expert_down on a given
 *     h_sorted [T*k][I] f32, which the kernel re-quantises to Q8_0 as the
 *     layer does; y_sorted [T*k][H] f32 output; acc [T*k][H][I/32] int32.
 * ws: at least qrx_workspace_bytes(cfg, T) bytes. */
int qrx_expert_gateup_q8_sums(const qrx_cfg *cfg, const qrx_experts *routed, const qrx_perm *perm,
                              const qrx_act *act, int32_t T, float *h_sorted, int32_t *acc,
                              void *ws, size_t ws_bytes, void *stream);
int qrx_expert_down_q8_sums(const qrx_cfg *cfg, const qrx_experts *routed, const qrx_perm *perm,
                            const float *h_sorted, int32_t T, float *y_sorted, int32_t *acc,
                            void *ws, size_t ws_bytes, void *stream);

/* Shared expert (README "已实现的功能"): the same FFN on every token, weight
 * 1, ungated.  h_sh [T][I] (may be NULL), y_sh [T][H] f32. */
int qrx_shared_ffn(const qrx_cfg *cfg, const qrx_experts *shared, const qrx_act *act,
                   int32_t T, float *h_sh, float *y_sh, void *ws, size_t ws_bytes,
                   void *stream);

/* Weighted combine (README "JustVugg/colibri", section "已实现的功能": routed
 * experts weighted by the router, plus the shared expert):
 * out[t] = y_sh[t] + sum_j topk_w[t][j] * y_sorted[inv[t*k+j]]
 * in fixed j order.  y_sh may be NULL (no shared term).  A slot with
 * inv < 0 (dropped by adaptive top-p) contributes nothing, whatever its
 * weight.  out [T][H] f32. */
int qrx_combine(const qrx_cfg *cfg, const float *y_sorted, const float *y_sh,
                const float *topk_w, const int32_t *inv, int32_t T, float *out,
                void *stream);

/* qrx_expert_ffn without any caller workspace, for callers that cannot
 * allocate device memory when they call in: for example a host whose memory
 * allocator owns the whole device budget and hands out nothing after start-up,
 * or a plug-in loaded into another runtime that gives it no allocator and no
 * workspace.  There is no counterpart of this call on the colibri pages; it is
 * the routed FFN of qrx_expert_ffn with its scratch (the gate/up output h,
 * T*k*I f32 values, and the digit records of the activations and of h) held
 * in a fixed 8 MiB array inside the library.
 *   - Limit: the 256-byte-aligned T*top_k*inter*4 bytes of h, plus T records
 *     of the activations and T*top_k records of h must fit 8 MiB.  A record of
 *     a row of length K takes 3*K + 16*(K/32) bytes (f32, bf16) or
 *     K + 8*(K/32) bytes (Q8_0).  For the GLM shape (H = 6144, I = 2048,
 *     k = 8) that is T <= 58 with f32 or bf16 activations.  Larger T returns
 *     QRX_ENOSPACE before any launch.
 *   - The array is a file-scope device variable: every GPU that loads the
 *     library holds its 8 MiB until the process exits.  Every call looks up
 *     the array's device address in the current device's context
 *     (cudaGetSymbolAddress, which allocates nothing), so the address stays
 *     right after cudaDeviceReset or in another context.  The first call on a
 *     device may load the library's kernels into that device's context: make
 *     it before any stream capture.
 *   - The array is shared by all calls on a device and keeps the last call's
 *     contents; nothing in it needs clearing, because every record and every
 *     row of h that a kernel reads is written by the same call first.  Calls
 *     that overlap on the GPU (on different streams, or from different host
 *     threads) race on the array: serialise them.
 *   - The call allocates nothing (no cudaMalloc, no library allocation).
 * Arguments and results are as qrx_expert_ffn, minus h_sorted and ws. */
int qrx_expert_ffn_noalloc(const qrx_cfg *cfg, const qrx_experts *routed,
                           const qrx_perm *perm, const qrx_act *act, int32_t T,
                           float *y_sorted, void *stream);

/* ---- the whole layer --------------------------------------------------- */

/* route -> permute -> routed + shared FFN -> combine (README "JustVugg/colibri",
 * section "已实现的功能": the router, the batch-union MoE, the shared expert),
 * all on `stream` with no host synchronisation.  (Capture into a CUDA graph
 * is not tested; the first call on a device also raises kernels' shared-memory
 * limits, so make one call before capturing.)
 * The kernels after the first are chained with programmatic dependent launch:
 * each may start while its predecessor drains and waits for it only where it
 * reads its output.
 * shared may be NULL.  x: the activations in cfg->afmt (f32 or bf16 [T][H];
 * Q8_0 is quantised from f32 x inside the call), 16-byte aligned.
 * topk_idx, topk_w: outputs [T][k].  out [T][H] f32, 16-byte aligned.
 * Expert FFN engines, by the call's shape:
 *   T = 1: the decode GEMV; its gate/up launch also makes the selection and
 *          the permutation from the router logits, its down launch also the
 *          combine (three launches in all);
 *   2 <= T <= 64 with int4 / int8 experts (int2: with f32 / bf16
 *          activations): the multi-token GEMV, the dot products on tensor
 *          cores (mma.sync, 8-bit codes x 8-bit digits -> exact int32);
 *   bf16 activations, int4 experts, T >= 256, H and I multiples of 256:
 *          grouped GEMMs on the tcgen05 tensor cores (bf16 x bf16 -> f32;
 *          int4 codes are exact in bf16);
 *   otherwise: the HBM-streaming dp4a GEMV. */
int qrx_moe_forward(const qrx_cfg *cfg, const void *x, int32_t T, const float *W_router,
                    const float *bias, const qrx_experts *routed, const qrx_experts *shared,
                    int32_t *topk_idx, float *topk_w, float *out, void *ws,
                    size_t ws_bytes, void *stream);

/* Options of qrx_moe_forward_opts. */
typedef struct {
    float expert_top_p;   /* adaptive expert top-p (see qrx_topp_prune), applied
                             inside the router's selection kernel; 0: off */
    uint64_t *usage;      /* [E] device usage counters (see qrx_usage_accumulate),
                             updated inside the permutation kernel; NULL: off */
} qrx_moe_opts;

/* qrx_moe_forward with options (opts may be NULL: same as qrx_moe_forward).
 * With top-p on, dropped slots come back as topk_idx = -1, topk_w = 0 and
 * take no part in the union, the expert FFN or the combine.  Neither option
 * adds a kernel launch.  QRX_EINVAL for a NaN top-p or a misaligned usage. */
int qrx_moe_forward_opts(const qrx_cfg *cfg, const void *x, int32_t T, const float *W_router,
                         const float *bias, const qrx_experts *routed, const qrx_experts *shared,
                         int32_t *topk_idx, float *topk_w, float *out, void *ws, size_t ws_bytes,
                         const qrx_moe_opts *opts, void *stream);

/* qrx_moe_forward with stage timing: events[0..6] are cudaEvent_t handles
 * (passed as void*) recorded on `stream` before the activation-record
 * kernel, after it (the two coincide when the expert engine builds its own
 * records), after the router, after the permutation, after the gate/up
 * kernel, after the down kernel and after the combine.  For batches of up to
 * 32 tokens the expert selection runs in the permutation's kernel, so
 * "router" is the logits kernel and "permutation" the selection with it.  n_events must
 * be 7.  The events separate the kernels, so the launch overlap that
 * qrx_moe_forward gets from programmatic dependent launch is lost here: the
 * stage times add up to more than a plain call takes.  opts as in
 * qrx_moe_forward_opts (may be NULL).  Everything else is as qrx_moe_forward. */
int qrx_moe_forward_profiled(const qrx_cfg *cfg, const void *x, int32_t T,
                             const float *W_router, const float *bias,
                             const qrx_experts *routed, const qrx_experts *shared,
                             int32_t *topk_idx, float *topk_w, float *out, void *ws,
                             size_t ws_bytes, void *const *events, int32_t n_events,
                             const qrx_moe_opts *opts, void *stream);

/* The same layer with HOST input and output: copies x_host (pinned or
 * pageable, T*H elements of the activation type) to the device, runs
 * qrx_moe_forward and copies the result to out_host [T][H] f32, then
 * synchronises `stream`.  ws must also hold the device copies:
 * qrx_workspace_bytes(cfg, T) covers them. */
int qrx_moe_forward_hostio(const qrx_cfg *cfg, const void *x_host, int32_t T,
                           const float *W_router, const float *bias,
                           const qrx_experts *routed, const qrx_experts *shared,
                           float *out_host, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QRX_H */
