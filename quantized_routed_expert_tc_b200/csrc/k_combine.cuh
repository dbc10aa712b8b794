// k_combine.cuh -- weighted combine of the routed expert outputs with the
// shared expert: out[t] = y_sh[t] + sum_j w[t, j] * y_sorted[inv[t*k + j]],
// j in ascending order (README "JustVugg/colibri", "已实现的功能": routed
// experts plus a shared expert; weights from the router).
#pragma once
#include "qrx_dev.cuh"
#include "qrx_check.cuh"

namespace qrx {

// One thread per 4 consecutive outputs of one token.
__global__ void __launch_bounds__(256) k_combine(const float *__restrict__ y, const float *__restrict__ ysh,
                                                 const float *__restrict__ w,
                                                 const int32_t *__restrict__ inv, int T, int k, int H,
                                                 float *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int hq = H / 4;
    if (id >= (int64_t)T * hq) return;
    const int t = (int)(id / hq), h = (int)(id % hq) * 4;
    float4 acc = ysh ? *reinterpret_cast<const float4 *>(ysh + (int64_t)t * H + h)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int64_t a = (int64_t)t * k + j;
        const float wj = w[a];
        const int p = inv[a];
        if (p < 0) continue;
        QRX_CHECK_OR(p < (int64_t)T * k, continue);
        const float4 v = *reinterpret_cast<const float4 *>(y + (int64_t)p * H + h);
        acc.x = fmaf(wj, v.x, acc.x);
        acc.y = fmaf(wj, v.y, acc.y);
        acc.z = fmaf(wj, v.z, acc.z);
        acc.w = fmaf(wj, v.w, acc.w);
    }
    *reinterpret_cast<float4 *>(out + (int64_t)t * H + h) = acc;
}

cudaError_t launch_combine(const float *y_sorted, const float *y_sh, const float *w,
                           const int32_t *inv, int T, int k, int H, float *out, cudaStream_t st)
{
    const int64_t n = (int64_t)T * (H / 4);
    return launch_k(k_combine, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, y_sorted, y_sh, w,
                    inv, T, k, H, out);
}

}  // namespace qrx
