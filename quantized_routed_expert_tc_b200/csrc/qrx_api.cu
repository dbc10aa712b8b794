// qrx_api.cu -- the C ABI of libqrx (declared in include/qrx.h) and the
// single translation unit that holds every kernel of the library.
//
// The calls follow the statement of the routed-MoE layer on the colibri pages
// (README "JustVugg/colibri", section "已实现的功能"): route, build the batch
// union, run the experts' quantised SwiGLU FFNs over it, add the shared
// expert, combine.  Every step runs in the kernels included below; the host
// code only checks arguments, carves the caller's workspace and launches.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "qrx_internal.h"
#include "qrx_dev.cuh"
#include "k_quant.cuh"
#include "k_permute.cuh"
#include "k_router.cuh"
#include "k_ffn_gemv.cuh"
#include "k_ffn_tc.cuh"
#include "k_gemv2.cuh"
#include "k_gmma.cuh"
#include "k_combine.cuh"

using namespace qrx;

thread_local bool qrx::g_pdl = false;

namespace {

// Sets the programmatic-dependent-launch switch for the launches in its scope.
struct PdlScope {
    explicit PdlScope(bool on) { g_pdl = on; }
    ~PdlScope() { g_pdl = false; }
};

constexpr int kMaxDevices = 64;

int num_sms_current()
{
    // per device, 0 until first asked; threads that race all store the same value
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

bool chunks_ok(int64_t K, int wbits)
{
    const int64_t cpr = K * wbits / 128;
    static const int allowed[] = {1, 2, 4, 8, 16, 32, 64, 96, 128, 192, 384};
    if (K * wbits % 128 != 0) return false;
    for (int a : allowed)
        if (cpr == a) return true;
    return false;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Workspace regions for T tokens.
struct Ws {
    size_t logits, counts, offsets, sorted, inv, uids, nu, xq, xd, xrec, hrec, xperm, hperm, h, y,
        xdev, outdev, idx, w, g2tab, g2cnt, g2hmax, rpart, rcnt, total;
};

Ws ws_layout(const qrx_cfg *c, int T)
{
    Ws L{};
    const int64_t E = c->n_experts, H = c->hidden, I = c->inter, k = c->top_k;
    const int64_t A = (int64_t)T * k;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.logits = take((size_t)T * E * sizeof(float));
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.sorted = take(A * 4);
    L.inv = take(A * 4);
    L.uids = take(E * 4);
    L.nu = take(4);
    L.xq = take((size_t)T * H);
    L.xd = take((size_t)T * (H / 32) * 4);
    L.xrec = take(act_records_bytes(c->afmt, (int)H, T));
    L.hrec = take(act_records_bytes(c->afmt, (int)I, (int)(A + T)));
    L.xperm = take((size_t)(A + T) * H * 2);     // tokens gathered in expert order, then in order
    L.hperm = take((size_t)(A + T) * I * 2);
    L.h = take((size_t)(A + T) * I * 4);
    L.y = take((size_t)(A + T) * H * 4);
    L.xdev = take((size_t)T * H * 4);
    L.outdev = take((size_t)T * H * 4);
    L.idx = take(A * 4);
    L.w = take(A * 4);
    L.g2tab = take((size_t)(4 + 4 * (std::min<int64_t>(E, A) + 1)) * 4);   // decode path: slot table
    L.g2cnt = take((size_t)H * 4);                                          // decode path: combine counters
    L.g2hmax = take((size_t)(A + T) * 4);                                   // decode path: largest |h| per row
    {
        const int ns = router_slices(T, (int)E, (int)H);
        L.rpart = take(ns > 1 ? (size_t)ns * T * E * 8 : 8);                 // router split-K partials
    }
    L.rcnt = take((size_t)((E + 63) / 64) * ((T + 63) / 64) * 4);          // router split-K tile counters
    L.total = off;
    return L;
}

template <typename Tp>
Tp *at(void *ws, size_t off)
{
    return reinterpret_cast<Tp *>(static_cast<char *>(ws) + off);
}

int cuda_code(cudaError_t e) { return e == cudaSuccess ? QRX_OK : QRX_ECUDA; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_common(const qrx_cfg *c, int T)
{
    int v = qrx_validate(c);
    if (v != QRX_OK) return v;
    if (T <= 0 || (int64_t)T * c->top_k > (1 << 26)) return QRX_EINVAL;
    return QRX_OK;
}

int check_ws(const qrx_cfg *c, int T, void *ws, size_t ws_bytes)
{
    if (!ws) return QRX_EINVAL;
    if (!aligned(ws, 256)) return QRX_EINVAL;
    if (ws_bytes < ws_layout(c, T).total) return QRX_ENOSPACE;
    return QRX_OK;
}

// One packed matrix: pointers 16-byte aligned; for a set of several experts
// the strides keep every expert's codes and scales 16-byte aligned.
int check_mat(const qrx_mat &m, bool several)
{
    if (!m.q || !m.scale || !aligned(m.q, 16) || !aligned(m.scale, 16)) return QRX_EINVAL;
    if (several && (m.expert_stride_q < 0 || m.expert_stride_q % 16 != 0 || m.expert_stride_q >= ((int64_t)1 << 40) ||
                    m.expert_stride_s < 0 || m.expert_stride_s % 4 != 0))
        return QRX_EINVAL;
    return QRX_OK;
}

int check_experts(const qrx_experts *x, bool several = true)
{
    if (!x) return QRX_EINVAL;
    int v;
    if ((v = check_mat(x->gate, several)) || (v = check_mat(x->up, several)) || (v = check_mat(x->down, several)))
        return v;
    return QRX_OK;
}

MatRef mat_ref(const qrx_mat &m) { return MatRef{m.q, m.scale, m.expert_stride_q, m.expert_stride_s}; }

int check_act(const qrx_cfg *c, const qrx_act *a)
{
    if (!a) return QRX_EINVAL;
    if (c->afmt == QRX_A_Q8_0)
        return (a->xq && a->xd && aligned(a->xq, 16) && aligned(a->xd, 16)) ? QRX_OK : QRX_EINVAL;
    return (a->x && aligned(a->x, 16)) ? QRX_OK : QRX_EINVAL;
}

int check_perm(const qrx_perm *p)
{
    if (!p || !p->counts || !p->offsets || !p->sorted || !p->inv || !p->union_ids || !p->n_union)
        return QRX_EINVAL;
    return QRX_OK;
}

FfnArgs ffn_args(const qrx_cfg *c, int T)
{
    FfnArgs a{};
    a.wbits = c->wfmt;
    a.afmt = c->afmt;
    a.H = c->hidden;
    a.I = c->inter;
    a.E = c->n_experts;
    a.k = c->top_k;
    a.T = T;
    return a;
}

void set_act(FfnArgs &a, const qrx_act *act)
{
    a.x = act->x;
    a.xq = act->xq;
    a.xd = act->xd;
}

void set_routed(FfnArgs &a, const qrx_experts *r, const qrx_perm *p)
{
    a.routed = 1;
    a.gate = mat_ref(r->gate);
    a.up = mat_ref(r->up);
    a.down = mat_ref(r->down);
    a.offsets = p->offsets;
    a.sorted = p->sorted;
    a.union_ids = p->union_ids;
    a.n_union = p->n_union;
}

void set_shared(FfnArgs &a, const qrx_experts *s)
{
    a.shared = 1;
    a.gate_sh = mat_ref(s->gate);
    a.up_sh = mat_ref(s->up);
    a.down_sh = mat_ref(s->down);
}

}  // namespace

extern "C" {

int qrx_validate(const qrx_cfg *c)
{
    if (!c) return QRX_EINVAL;
    if (c->hidden <= 0 || c->n_experts <= 0 || c->inter <= 0 || c->n_group <= 0 ||
        c->topk_group <= 0 || c->top_k <= 0)
        return QRX_EINVAL;
    if (c->wfmt != QRX_W_INT8 && c->wfmt != QRX_W_INT4 && c->wfmt != QRX_W_INT2) return QRX_EINVAL;
    if (c->afmt != QRX_A_F32 && c->afmt != QRX_A_Q8_0 && c->afmt != QRX_A_BF16) return QRX_EINVAL;
    if (!std::isfinite(c->routed_scaling_factor)) return QRX_EINVAL;
    if (c->n_experts % c->n_group != 0) return QRX_EUNSUPPORTED;
    if (c->topk_group > c->n_group) return QRX_EUNSUPPORTED;
    if ((int64_t)c->topk_group * (c->n_experts / c->n_group) < c->top_k) return QRX_EUNSUPPORTED;
    if (c->top_k > 32 || c->n_experts > 1024) return QRX_EUNSUPPORTED;
    if (c->hidden % 64 != 0 || c->inter % 64 != 0) return QRX_EUNSUPPORTED;
    if (!chunks_ok(c->hidden, c->wfmt) || !chunks_ok(c->inter, c->wfmt)) return QRX_EUNSUPPORTED;
    return QRX_OK;
}

size_t qrx_workspace_bytes(const qrx_cfg *c, int32_t T)
{
    if (qrx_validate(c) != QRX_OK || T <= 0) return 0;
    return ws_layout(c, T).total;
}

int qrx_ffn_engine(const qrx_cfg *c, int32_t T)
{
    if (qrx_validate(c) != QRX_OK || T <= 0) return QRX_EINVAL;
    return tc_shape_ok(c->afmt, c->wfmt, T, c->hidden, c->inter) ? QRX_ENGINE_TC : QRX_ENGINE_GEMV;
}

int qrx_last_error(void)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return QRX_ECUDA;
    int flag = 0;
    e = cudaMemcpyFromSymbol(&flag, g_status, sizeof(int));
    if (e != cudaSuccess) return QRX_ECUDA;
    if (flag != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
        if (e != cudaSuccess) return QRX_ECUDA;
    }
    if (flag == DERR_TIMEOUT) return QRX_ETIMEOUT;
    return flag ? QRX_EDEVICE : QRX_OK;
}

const char *qrx_strerror(int code)
{
    switch (code) {
    case QRX_OK: return "ok";
    case QRX_EINVAL: return "invalid argument";
    case QRX_EUNSUPPORTED: return "unsupported configuration";
    case QRX_ECUDA: return "CUDA runtime error";
    case QRX_ETIMEOUT: return "bounded device wait gave up";
    case QRX_EDEVICE: return "a kernel saw an invalid value";
    case QRX_ENOSPACE: return "workspace too small";
    default: return "unknown error";
    }
}

int qrx_quantize_weights(const float *w, int64_t rows, int64_t K, int32_t wbits, uint8_t *q,
                         int64_t ldq, float *scale, int64_t lds, void *stream)
{
    if (!w || !q || !scale || rows <= 0 || K <= 0 || K % 32 != 0) return QRX_EINVAL;
    if (wbits != 8 && wbits != 4 && wbits != 2) return QRX_EINVAL;
    if (ldq < K * wbits / 8 || ldq % 4 != 0 || lds < 1) return QRX_EINVAL;
    if (!aligned(w, 16) || !aligned(q, 4) || !aligned(scale, 4)) return QRX_EINVAL;
    return cuda_code(launch_quantize_weights(w, rows, K, wbits, q, ldq, scale, lds,
                                             (cudaStream_t)stream));
}

int qrx_requant_fp8(const uint8_t *w8, int64_t rows, int64_t K, int64_t ld8, const float *bscale,
                    int32_t wbits, uint8_t *q, int64_t ldq, float *scale, int64_t lds, void *stream)
{
    if (!w8 || !bscale || !q || !scale || rows <= 0 || K <= 0 || K % 32 != 0) return QRX_EINVAL;
    if (wbits != 8 && wbits != 4 && wbits != 2) return QRX_EINVAL;
    if (ld8 < K || ld8 % 4 != 0 || ldq < K * wbits / 8 || ldq % 4 != 0 || lds < 1) return QRX_EINVAL;
    if (!aligned(w8, 4) || !aligned(bscale, 4) || !aligned(q, 4) || !aligned(scale, 4)) return QRX_EINVAL;
    return cuda_code(launch_requant_fp8(w8, rows, K, ld8, bscale, wbits, q, ldq, scale, lds,
                                        (cudaStream_t)stream));
}

int qrx_quantize_act_q8(const float *x, int64_t T, int64_t H, int8_t *xq, float *xd, void *stream)
{
    if (!x || !xq || !xd || T <= 0 || H <= 0 || H % 32 != 0) return QRX_EINVAL;
    return cuda_code(launch_quantize_act_q8(x, T * H / 32, xq, xd, (cudaStream_t)stream));
}

int qrx_block_dots_q8(int32_t wbits, const uint8_t *q, int64_t rows, int64_t K, const int8_t *xq,
                      int32_t *acc, void *stream)
{
    if (!q || !xq || !acc || rows <= 0 || K <= 0 || K % 32 != 0) return QRX_EINVAL;
    if (wbits != 8 && wbits != 4 && wbits != 2) return QRX_EINVAL;
    if (!aligned(q, 4)) return QRX_EINVAL;
    return cuda_code(launch_block_dots_q8(wbits, q, rows, K, xq, acc, (cudaStream_t)stream));
}

// The router, with adaptive top-p applied in its select kernel when topp_thr > 0.
static RouterArgs router_args(const qrx_cfg *c, const void *x, int32_t T, const float *Wr, const float *bias,
                              int32_t *topk_idx, float *topk_w, void *ws, double topp_thr)
{
    const Ws L = ws_layout(c, T);
    RouterArgs a{};
    a.x = x;
    a.x_bf16 = c->afmt == QRX_A_BF16;
    a.Wr = Wr;
    a.bias = bias;
    a.T = T;
    a.H = c->hidden;
    a.E = c->n_experts;
    a.G = c->n_group;
    a.Gk = c->topk_group;
    a.k = c->top_k;
    a.rsf = c->routed_scaling_factor;
    a.logits = at<float>(ws, L.logits);
    a.part = at<double>(ws, L.rpart);
    a.tilecnt = at<int>(ws, L.rcnt);
    a.idx = topk_idx;
    a.w = topk_w;
    a.topp_thr = topp_thr;
    return a;
}

static int route_impl(const qrx_cfg *c, const void *x, int32_t T, const float *Wr, const float *bias,
                      int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream,
                      double topp_thr)
{
    int v = check_common(c, T);
    if (v) return v;
    if (!x || !Wr || !bias || !topk_idx || !topk_w) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    const RouterArgs a = router_args(c, x, T, Wr, bias, topk_idx, topk_w, ws, topp_thr);
    return cuda_code(launch_router(a, (cudaStream_t)stream));
}

// p * rsf for adaptive top-p, or 0 (off) when p is outside (0, 1).
static double topp_threshold(const qrx_cfg *c, float p)
{
    return (p > 0.f && p < 1.f) ? (double)p * (double)c->routed_scaling_factor : 0.0;
}

int qrx_route(const qrx_cfg *c, const void *x, int32_t T, const float *Wr, const float *bias,
              int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream)
{
    return route_impl(c, x, T, Wr, bias, topk_idx, topk_w, ws, ws_bytes, stream, 0.0);
}

int qrx_topp_prune(const qrx_cfg *c, int32_t *topk_idx, float *topk_w, int32_t T, float p, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if (!topk_idx || !topk_w || !(p == p)) return QRX_EINVAL;
    const double thr = topp_threshold(c, p);
    if (thr == 0.0) return QRX_OK;
    return cuda_code(launch_topp_prune(topk_idx, topk_w, T, c->top_k, thr, (cudaStream_t)stream));
}

int qrx_usage_accumulate(const qrx_cfg *c, const qrx_perm *perm, uint64_t *usage, void *stream)
{
    int v = qrx_validate(c);
    if (v) return v;
    if (!perm || !perm->counts || !usage || !aligned(usage, 8)) return QRX_EINVAL;
    return cuda_code(launch_usage_add(perm->counts, c->n_experts, usage, (cudaStream_t)stream));
}

int qrx_permute(const qrx_cfg *c, const int32_t *topk_idx, int32_t T, const qrx_perm *perm,
                void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if (!topk_idx || (v = check_perm(perm))) return v ? v : QRX_EINVAL;
    return cuda_code(launch_permute(topk_idx, T, c->top_k, c->n_experts, *perm, (cudaStream_t)stream));
}

int qrx_expert_ffn(const qrx_cfg *c, const qrx_experts *routed, const qrx_perm *perm,
                   const qrx_act *act, int32_t T, float *h_sorted, float *y_sorted, void *ws,
                   size_t ws_bytes, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(routed)) || (v = check_perm(perm)) || (v = check_act(c, act))) return v;
    if (!y_sorted) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    const Ws L = ws_layout(c, T);
    FfnArgs a = ffn_args(c, T);
    set_act(a, act);
    set_routed(a, routed, perm);
    a.h = h_sorted ? h_sorted : at<float>(ws, L.h);
    a.xrec = at<unsigned char>(ws, L.xrec);
    a.hrec = at<unsigned char>(ws, L.hrec);
    a.xperm = at<unsigned char>(ws, L.xperm);
    a.hperm = at<unsigned char>(ws, L.hperm);
    a.hperm_ready = 1;
    a.prep_records = 1;
    a.h_ld = c->inter;
    a.y = y_sorted;
    a.y_ld = c->hidden;
    if (!h_sorted && ffn_use_tc(a)) a.h = nullptr;   // down reads the bf16 copy of h
    const int sms = num_sms_current();
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_ffn_gateup(a, sms, st);
    if (e == cudaSuccess) e = launch_ffn_down(a, sms, st);
    return cuda_code(e);
}

int qrx_expert_down(const qrx_cfg *c, const qrx_experts *routed, const qrx_perm *perm,
                    const float *h_sorted, int32_t T, float *y_sorted, void *ws, size_t ws_bytes,
                    void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(routed)) || (v = check_perm(perm))) return v;
    if (!h_sorted || !y_sorted) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    FfnArgs a = ffn_args(c, T);
    set_routed(a, routed, perm);
    a.hrec = at<unsigned char>(ws, ws_layout(c, T).hrec);
    a.xperm = at<unsigned char>(ws, ws_layout(c, T).xperm);
    a.hperm = at<unsigned char>(ws, ws_layout(c, T).hperm);
    a.hperm_ready = 0;
    a.h = const_cast<float *>(h_sorted);
    a.h_ld = c->inter;
    a.y = y_sorted;
    a.y_ld = c->hidden;
    return cuda_code(launch_ffn_down(a, num_sms_current(), (cudaStream_t)stream));
}

int qrx_expert_gateup_q8_sums(const qrx_cfg *c, const qrx_experts *routed, const qrx_perm *perm,
                              const qrx_act *act, int32_t T, float *h_sorted, int32_t *acc, void *ws,
                              size_t ws_bytes, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(routed)) || (v = check_perm(perm)) || (v = check_act(c, act))) return v;
    if (!h_sorted || !acc) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    FfnArgs a = ffn_args(c, T);
    set_act(a, act);
    set_routed(a, routed, perm);
    if (c->afmt != QRX_A_Q8_0 || !g2_use(a)) return QRX_EUNSUPPORTED;
    a.h = h_sorted;
    a.h_ld = c->inter;
    return cuda_code(launch_g2_gateup(a, num_sms_current(), (cudaStream_t)stream, acc));
}

int qrx_expert_down_q8_sums(const qrx_cfg *c, const qrx_experts *routed, const qrx_perm *perm,
                            const float *h_sorted, int32_t T, float *y_sorted, int32_t *acc, void *ws,
                            size_t ws_bytes, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(routed)) || (v = check_perm(perm))) return v;
    if (!h_sorted || !y_sorted || !acc) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    FfnArgs a = ffn_args(c, T);
    set_routed(a, routed, perm);
    if (c->afmt != QRX_A_Q8_0 || !g2_use(a)) return QRX_EUNSUPPORTED;
    a.h = const_cast<float *>(h_sorted);
    a.h_ld = c->inter;
    a.y = y_sorted;
    a.y_ld = c->hidden;
    return cuda_code(launch_g2_down(a, num_sms_current(), (cudaStream_t)stream, acc));
}

int qrx_shared_ffn(const qrx_cfg *c, const qrx_experts *shared, const qrx_act *act, int32_t T,
                   float *h_sh, float *y_sh, void *ws, size_t ws_bytes, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(shared, false)) || (v = check_act(c, act))) return v;
    if (!y_sh) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    const Ws L = ws_layout(c, T);
    FfnArgs a = ffn_args(c, T);
    set_act(a, act);
    set_shared(a, shared);
    a.h = h_sh ? h_sh : at<float>(ws, L.h);
    a.xrec = at<unsigned char>(ws, L.xrec);
    a.hrec = at<unsigned char>(ws, L.hrec);
    a.xperm = at<unsigned char>(ws, L.xperm);
    a.hperm = at<unsigned char>(ws, L.hperm);
    a.hperm_ready = 1;
    a.prep_records = 1;
    a.h_ld = c->inter;
    a.y = y_sh;
    a.y_ld = c->hidden;
    a.sh_h_row0 = 0;
    a.sh_y_row0 = 0;
    const int sms = num_sms_current();
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_ffn_gateup(a, sms, st);
    if (e == cudaSuccess) e = launch_ffn_down(a, sms, st);
    return cuda_code(e);
}

int qrx_combine(const qrx_cfg *c, const float *y_sorted, const float *y_sh, const float *topk_w,
                const int32_t *inv, int32_t T, float *out, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if (!y_sorted || !topk_w || !inv || !out) return QRX_EINVAL;
    if (!aligned(y_sorted, 16) || !aligned(out, 16) || (y_sh && !aligned(y_sh, 16))) return QRX_EINVAL;
    return cuda_code(launch_combine(y_sorted, y_sh, topk_w, inv, T, c->top_k, c->hidden, out,
                                    (cudaStream_t)stream));
}

}  // extern "C"

namespace {

int moe_forward_impl(const qrx_cfg *c, const void *x, int32_t T, const float *Wr,
                     const float *bias, const qrx_experts *routed, const qrx_experts *shared,
                     int32_t *topk_idx, float *topk_w, float *out, void *ws, size_t ws_bytes,
                     void *const *events, void *stream, const qrx_moe_opts *opts = nullptr)
{
    auto mark = [&](int i) -> bool {
        return !events || cudaEventRecord((cudaEvent_t)events[i], (cudaStream_t)stream) == cudaSuccess;
    };
    int v = check_common(c, T);
    if (v) return v;
    if (!x || !Wr || !bias || !topk_idx || !topk_w || !out) return QRX_EINVAL;
    if (!aligned(x, 16)) return QRX_EINVAL;
    if ((v = check_experts(routed))) return v;
    if (shared && (v = check_experts(shared, false))) return v;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    if (!aligned(out, 16)) return QRX_EINVAL;
    if (opts && (!(opts->expert_top_p == opts->expert_top_p) || (opts->usage && !aligned(opts->usage, 8))))
        return QRX_EINVAL;
    const double topp_thr = opts ? topp_threshold(c, opts->expert_top_p) : 0.0;
    uint64_t *usage = opts ? opts->usage : nullptr;
    const Ws L = ws_layout(c, T);
    cudaStream_t st = (cudaStream_t)stream;
    const int sms = num_sms_current();
    const int64_t A = (int64_t)T * c->top_k;

    // 1. activation records (reads only x; ordinary stream order with what came before)
    FfnArgs a = ffn_args(c, T);
    a.x = x;                      // Q8_0: the records kernel quantises x itself
    a.xrec = at<unsigned char>(ws, L.xrec);
    a.hrec = at<unsigned char>(ws, L.hrec);
    a.xperm = at<unsigned char>(ws, L.xperm);
    a.hperm = at<unsigned char>(ws, L.hperm);
    a.hperm_ready = 1;
    if (!mark(0)) return QRX_ECUDA;
    // the tensor-core path needs no digit records; the decode GEMV builds its own
    const bool tc = ffn_use_tc(a), own_records = tc || g2_use(a) || gm_use(a);
    cudaError_t e = own_records ? cudaSuccess : launch_act_digits(a, st);
    if (e != cudaSuccess || !mark(1)) return QRX_ECUDA;
    // 2.. the rest chained with programmatic dependent launch (the first kernel
    // of the call never is: it must follow whatever the stream held before)
    PdlScope pdl(!own_records);
    qrx_perm perm{at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.sorted),
                  at<int32_t>(ws, L.inv), at<int32_t>(ws, L.uids), at<int32_t>(ws, L.nu)};
    const RouterArgs ra = router_args(c, x, T, Wr, bias, topk_idx, topk_w, ws, topp_thr);
    float *h = at<float>(ws, L.h), *y = at<float>(ws, L.y);
    set_routed(a, routed, &perm);
    if (shared) set_shared(a, shared);
    a.prep_records = 0;
    a.h = tc ? nullptr : h;       // the tensor-core down projection reads the bf16 copy of h
    a.h_ld = c->inter;
    a.y = y;
    a.y_ld = c->hidden;
    a.sh_h_row0 = A;
    a.sh_y_row0 = A;
    // decode GEMV: the gate/up kernel also selects and permutes, the down kernel also combines
    if (!tc && T == 1 && g2_fuse_ok(a, c->n_group, c->topk_group)) {
        RouterArgs rz = ra;
        rz.zero = at<uint32_t>(ws, L.g2hmax);
        rz.nzero = (int)(A + T);
        e = launch_router(rz, st, false);
        g_pdl = true;
        if (e != cudaSuccess || !mark(2) || !mark(3)) return QRX_ECUDA;
        G2Fuse f{};
        f.logits = ra.logits;
        f.bias = bias;
        f.G = c->n_group;
        f.Gk = c->topk_group;
        f.rsf = c->routed_scaling_factor;
        f.topp_thr = topp_thr;
        f.idx = topk_idx;
        f.w = topk_w;
        f.usage = usage;
        f.counts = perm.counts;
        f.inv = perm.inv;
        f.tab = at<int32_t>(ws, L.g2tab);
        f.cnt = at<int32_t>(ws, L.g2cnt);
        f.out = out;
        f.hmax = rz.zero;
        e = launch_g2_gateup_fused(a, f, sms, st);
        if (e != cudaSuccess || !mark(4)) return QRX_ECUDA;
        e = launch_g2_down_fused(a, f, sms, st);
        if (e != cudaSuccess || !mark(5) || !mark(6)) return QRX_ECUDA;
        return QRX_OK;
    }
    // small batches: selection and permutation in one kernel after the logits
    const bool fused = select_permute_fused_ok(T, c->n_experts, c->n_group);
    e = launch_router(ra, st, !fused);
    g_pdl = true;
    if (e != cudaSuccess || !mark(2)) return QRX_ECUDA;
    e = fused ? launch_select_permute(ra, perm, usage, st)
              : launch_permute(topk_idx, T, c->top_k, c->n_experts, perm, st, usage);
    if (e != cudaSuccess || !mark(3)) return QRX_ECUDA;
    e = launch_ffn_gateup(a, sms, st);
    if (e != cudaSuccess || !mark(4)) return QRX_ECUDA;
    e = launch_ffn_down(a, sms, st);
    if (e != cudaSuccess || !mark(5)) return QRX_ECUDA;
    e = launch_combine(y, shared ? y + A * c->hidden : nullptr, topk_w, perm.inv, T, c->top_k,
                       c->hidden, out, st);
    if (e != cudaSuccess || !mark(6)) return QRX_ECUDA;
    return QRX_OK;
}

}  // namespace

extern "C" {

int qrx_moe_forward(const qrx_cfg *c, const void *x, int32_t T, const float *Wr, const float *bias,
                    const qrx_experts *routed, const qrx_experts *shared, int32_t *topk_idx,
                    float *topk_w, float *out, void *ws, size_t ws_bytes, void *stream)
{
    return moe_forward_impl(c, x, T, Wr, bias, routed, shared, topk_idx, topk_w, out, ws, ws_bytes,
                            nullptr, stream);
}

int qrx_moe_forward_opts(const qrx_cfg *c, const void *x, int32_t T, const float *Wr,
                         const float *bias, const qrx_experts *routed, const qrx_experts *shared,
                         int32_t *topk_idx, float *topk_w, float *out, void *ws, size_t ws_bytes,
                         const qrx_moe_opts *opts, void *stream)
{
    return moe_forward_impl(c, x, T, Wr, bias, routed, shared, topk_idx, topk_w, out, ws, ws_bytes,
                            nullptr, stream, opts);
}

int qrx_moe_forward_profiled(const qrx_cfg *c, const void *x, int32_t T, const float *Wr,
                             const float *bias, const qrx_experts *routed,
                             const qrx_experts *shared, int32_t *topk_idx, float *topk_w,
                             float *out, void *ws, size_t ws_bytes, void *const *events,
                             int32_t n_events, const qrx_moe_opts *opts, void *stream)
{
    if (!events || n_events != 7) return QRX_EINVAL;
    for (int i = 0; i < 7; ++i)
        if (!events[i]) return QRX_EINVAL;
    return moe_forward_impl(c, x, T, Wr, bias, routed, shared, topk_idx, topk_w, out, ws, ws_bytes,
                            events, stream, opts);
}

int qrx_moe_forward_hostio(const qrx_cfg *c, const void *x_host, int32_t T, const float *Wr,
                           const float *bias, const qrx_experts *routed, const qrx_experts *shared,
                           float *out_host, void *ws, size_t ws_bytes, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if (!x_host || !out_host) return QRX_EINVAL;
    if ((v = check_ws(c, T, ws, ws_bytes))) return v;
    const Ws L = ws_layout(c, T);
    cudaStream_t st = (cudaStream_t)stream;
    const size_t xbytes = (size_t)T * c->hidden * (c->afmt == QRX_A_BF16 ? 2 : 4);
    void *xdev = at<char>(ws, L.xdev);
    float *odev = at<float>(ws, L.outdev);
    if (cudaMemcpyAsync(xdev, x_host, xbytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return QRX_ECUDA;
    v = qrx_moe_forward(c, xdev, T, Wr, bias, routed, shared, at<int32_t>(ws, L.idx),
                        at<float>(ws, L.w), odev, ws, ws_bytes, stream);
    if (v) return v;
    if (cudaMemcpyAsync(out_host, odev, (size_t)T * c->hidden * 4, cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
        return QRX_ECUDA;
    return cuda_code(cudaStreamSynchronize(st));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free routed FFN: its scratch (h) lives in a fixed device array.
// Callers that cannot allocate device memory when they call in use this entry
// point instead of qrx_expert_ffn.  The array's name is only a host-side
// handle in host code; its device address comes from cudaGetSymbolAddress,
// looked up once per device with that device current.
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;   // 8 MiB per device

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// The array's device address in the current device's context.  Looked up on
// every call: the lookup allocates nothing, and a cached address could be
// stale after cudaDeviceReset or in another context on the same device.
int noalloc_scratch(void **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QRX_ECUDA;
    *out = p;
    return QRX_OK;
}

}  // namespace

extern "C" int qrx_expert_ffn_noalloc(const qrx_cfg *c, const qrx_experts *routed,
                                      const qrx_perm *perm, const qrx_act *act, int32_t T,
                                      float *y_sorted, void *stream)
{
    int v = check_common(c, T);
    if (v) return v;
    if ((v = check_experts(routed)) || (v = check_perm(perm)) || (v = check_act(c, act))) return v;
    if (!y_sorted) return QRX_EINVAL;
    const size_t hbytes = align256((size_t)T * c->top_k * c->inter * sizeof(float));
    const size_t xbytes = align256(act_records_bytes(c->afmt, c->hidden, T));
    const size_t need = hbytes + xbytes + act_records_bytes(c->afmt, c->inter, T * c->top_k);
    if (need > kNoAllocScratchBytes) return QRX_ENOSPACE;
    void *scratch = nullptr;
    if ((v = noalloc_scratch(&scratch))) return v;
    FfnArgs a = ffn_args(c, T);
    set_act(a, act);
    set_routed(a, routed, perm);
    a.h = static_cast<float *>(scratch);
    a.xrec = static_cast<unsigned char *>(scratch) + hbytes;
    a.hrec = static_cast<unsigned char *>(scratch) + hbytes + xbytes;
    a.prep_records = 1;
    a.h_ld = c->inter;
    a.y = y_sorted;
    a.y_ld = c->hidden;
    const int sms = num_sms_current();
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_ffn_gateup(a, sms, st);
    if (e == cudaSuccess) e = launch_ffn_down(a, sms, st);
    return cuda_code(e);
}
