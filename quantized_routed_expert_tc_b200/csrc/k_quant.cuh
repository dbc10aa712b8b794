// k_quant.cuh -- per-row weight quantiser, Q8_0 activation quantiser and the
// exact block-accumulator kernel.
//
// Per-row symmetric quantisation: README "JustVugg/colibri", section
// "已实现的功能" (int8 / packed int4 / packed int2 with per-row scales); the
// tiny-layer workload fixes scale = absmax/7 and "two per byte, low nibble
// first" for int4.  Q8_0: README "已实现的功能" (Q8_0-style int8
// activations), blocks of 32 with an f32 absmax scale.
#pragma once
#include "qrx_dev.cuh"

namespace qrx {

// One warp per row.  Pass 1: absmax.  Pass 2: codes, packed into 32-bit
// words (4, 8 or 16 codes per word), one word per lane per step.
template <int WB>
__global__ void __launch_bounds__(256) k_quantize_weights(const float *__restrict__ w, int64_t rows,
                                                          int64_t K, uint8_t *__restrict__ q,
                                                          int64_t ldq, float *__restrict__ scale,
                                                          int64_t lds)
{
    constexpr int QMAX = WB == 8 ? 127 : (WB == 4 ? 7 : 1);
    constexpr int QMIN = WB == 8 ? -128 : (WB == 4 ? -8 : -2);
    constexpr int EPW = 32 / WB;     // codes per 32-bit word
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const float *wr = w + r * K;
    float amax = 0.f;
    for (int64_t i = lane * 4; i < K; i += 128) {
        float4 v = *reinterpret_cast<const float4 *>(wr + i);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = warp_max(amax);
    const float s = __fdiv_rn(amax, (float)QMAX);
    if (lane == 0) scale[r * lds] = s;
    uint32_t *qr = reinterpret_cast<uint32_t *>(q + r * ldq);
    const int64_t nwords = K / EPW;
    for (int64_t wd = lane; wd < nwords; wd += 32) {
        const float *src = wr + wd * EPW;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < EPW; i += 4) {
            float4 v = *reinterpret_cast<const float4 *>(src + i);
            float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int c = 0;
                if (s != 0.f) {
                    c = (int)roundf(__fdiv_rn(vv[j], s));
                    c = c > QMAX ? QMAX : (c < QMIN ? QMIN : c);
                }
                word |= ((uint32_t)c & ((1u << WB) - 1u)) << (WB * (i + j));
            }
        }
        qr[wd] = word;
    }
}

// FP8 (e4m3, 128x128 block scales) -> per-row packed codes (README
// "JustVugg/colibri", section "已实现的功能": the FP8->int4 converter
// dequantises with 128x128 block scales and requantises into the per-row
// container).  One warp per row; each value is f32(fp8) * block scale (a NaN
// code counts as 0), recomputed in pass 2 instead of kept: the row's FP8
// bytes are re-read from L2.  Pass 1: absmax; pass 2: codes
// round-half-away(fl(x / s)).  Lanes read 4 codes at a time (K % 32 == 0,
// rows 4-byte aligned) and decode them in pairs.
//
// The quotient: t = x * (1/s) is within ~3 * 2^-24 (relative) of the
// correctly rounded fl(x / s), so when t is farther than 1e-6 * |t| from a
// half-integer both round to the same integer; only near a half-integer (or
// when 1/s is not finite) is the division itself computed.
__device__ __forceinline__ void fp8x4_values(uint32_t v, float sc, float (&f)[4])
{
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v >> 16), __NV_E4M3);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (f[j] != f[j]) f[j] = 0.f;
        f[j] = __fmul_rn(f[j], sc);
    }
}

__device__ __forceinline__ int requant_code(float x, float s, float inv, bool inv_ok, int qmin, int qmax)
{
    float r;
    const float t = __fmul_rn(x, inv);
    const float d = fabsf(t - floorf(t) - 0.5f);
    if (inv_ok && d > 1e-6f * fabsf(t)) r = t;
    else r = __fdiv_rn(x, s);
    int c = (int)roundf(r);
    return c > qmax ? qmax : (c < qmin ? qmin : c);
}

template <int WB>
__global__ void __launch_bounds__(256) k_requant_fp8(const uint8_t *__restrict__ w8, int64_t rows, int64_t K,
                                                     int64_t ld8, const float *__restrict__ bscale,
                                                     uint8_t *__restrict__ q, int64_t ldq,
                                                     float *__restrict__ scale, int64_t lds)
{
    constexpr int QMAX = WB == 8 ? 127 : (WB == 4 ? 7 : 1);
    constexpr int QMIN = WB == 8 ? -128 : (WB == 4 ? -8 : -2);
    constexpr int EPW = 32 / WB;     // codes per 32-bit word
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    pdl_wait();
    pdl_trigger();
    if (r >= rows) return;
    const uint8_t *wr = w8 + r * ld8;
    const float *bs = bscale + (r / 128) * ((K + 127) / 128);
    float amax = 0.f;
    for (int64_t i = lane * 4; i < K; i += 128) {
        float f[4];
        fp8x4_values(*reinterpret_cast<const uint32_t *>(wr + i), bs[i / 128], f);   // 4 columns, one block
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
    amax = warp_max(amax);
    const float s = __fdiv_rn(amax, (float)QMAX);
    const float inv = s != 0.f ? __frcp_rn(s) : 0.f;
    const bool inv_ok = s != 0.f && isfinite(inv);
    if (lane == 0) scale[r * lds] = s;
    uint32_t *qr = reinterpret_cast<uint32_t *>(q + r * ldq);
    const int64_t nwords = K / EPW;
    for (int64_t wd = lane; wd < nwords; wd += 32) {
        const int64_t c0 = wd * EPW;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < EPW; i += 4) {
            float f[4];
            fp8x4_values(*reinterpret_cast<const uint32_t *>(wr + c0 + i), bs[(c0 + i) / 128], f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = s != 0.f ? requant_code(f[j], s, inv, inv_ok, QMIN, QMAX) : 0;
                word |= ((uint32_t)c & ((1u << WB) - 1u)) << (WB * (i + j));
            }
        }
        qr[wd] = word;
    }
}

// One warp per 32-element block.
__global__ void __launch_bounds__(256) k_quantize_act_q8(const float *__restrict__ x, int64_t nblocks,
                                                         int8_t *__restrict__ xq,
                                                         float *__restrict__ xd)
{
    const int lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= nblocks) return;
    const float v = x[b * 32 + lane];
    const float amax = warp_max(fabsf(v));
    int c = 0;
    if (amax != 0.f) {
        c = q8_code(v, __fdiv_rn(127.f, amax));
    }
    xq[b * 32 + lane] = (int8_t)c;
    if (lane == 0) xd[b] = amax != 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
}

// Exact block accumulators through unpack_word + dp4a (the FFN kernels' path).
// One thread per (row, 32-element block).
template <int WB>
__global__ void __launch_bounds__(256) k_block_dots_q8(const uint8_t *__restrict__ q, int64_t rows,
                                                       int64_t K, const int8_t *__restrict__ xq,
                                                       int32_t *__restrict__ acc)
{
    using F = Fmt<WB>;
    const int64_t nb = K / 32;
    const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= rows * nb) return;
    const int64_t r = id / nb, b = id % nb;
    const int64_t rb = K * WB / 8;
    // the block's 32 codes are WB words; word wi of the block is word (wi % 4)
    // of chunk (block*32 + wi*EPW)/EPC
    constexpr int EPW = 32 / WB;
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(q + r * rb + b * 32 * WB / 8);
    int s = 0, xsum = 0;
    for (int wi = 0; wi < WB; ++wi) {
        const int64_t e0 = b * 32 + (int64_t)wi * EPW;          // first element of the word
        const int64_t chunk_base = (e0 / F::EPC) * F::EPC;
        const int iw = (int)((e0 - chunk_base) / EPW);           // word index within chunk
        uint32_t u[F::UPW];
        unpack_word<WB>(qw[wi], u);
#pragma unroll
        for (int j = 0; j < F::UPW; ++j) {
            uint32_t dw = 0;
#pragma unroll
            for (int by = 0; by < 4; ++by) {
                int8_t xv = xq[chunk_base + elem_in_chunk<WB>(iw, j, by)];
                dw |= (uint32_t)(uint8_t)xv << (8 * by);
                xsum += xv;
            }
            s = dp4a(u[j], dw, s);
        }
    }
    acc[id] = s - F::OFF * xsum;
}

cudaError_t launch_quantize_weights(const float *w, int64_t rows, int64_t K, int wbits,
                                    uint8_t *q, int64_t ldq, float *scale, int64_t lds,
                                    cudaStream_t st)
{
    const int wpb = 8;
    dim3 grid((unsigned)((rows + wpb - 1) / wpb)), block(32 * wpb);
    if (wbits == 8) k_quantize_weights<8><<<grid, block, 0, st>>>(w, rows, K, q, ldq, scale, lds);
    else if (wbits == 4) k_quantize_weights<4><<<grid, block, 0, st>>>(w, rows, K, q, ldq, scale, lds);
    else k_quantize_weights<2><<<grid, block, 0, st>>>(w, rows, K, q, ldq, scale, lds);
    return cudaGetLastError();
}

cudaError_t launch_requant_fp8(const uint8_t *w8, int64_t rows, int64_t K, int64_t ld8, const float *bscale,
                              int wbits, uint8_t *q, int64_t ldq, float *scale, int64_t lds, cudaStream_t st)
{
    const int wpb = 8;
    const dim3 grid((unsigned)((rows + wpb - 1) / wpb)), block(32 * wpb);
    if (wbits == 8) return launch_k(k_requant_fp8<8>, grid, block, 0, st, w8, rows, K, ld8, bscale, q, ldq, scale, lds);
    if (wbits == 4) return launch_k(k_requant_fp8<4>, grid, block, 0, st, w8, rows, K, ld8, bscale, q, ldq, scale, lds);
    return launch_k(k_requant_fp8<2>, grid, block, 0, st, w8, rows, K, ld8, bscale, q, ldq, scale, lds);
}

cudaError_t launch_quantize_act_q8(const float *x, int64_t nblocks, int8_t *xq, float *xd,
                                   cudaStream_t st)
{
    const int wpb = 8;
    k_quantize_act_q8<<<(unsigned)((nblocks + wpb - 1) / wpb), 32 * wpb, 0, st>>>(x, nblocks, xq, xd);
    return cudaGetLastError();
}

cudaError_t launch_block_dots_q8(int wbits, const uint8_t *q, int64_t rows, int64_t K,
                                 const int8_t *xq, int32_t *acc, cudaStream_t st)
{
    const int64_t n = rows * (K / 32);
    dim3 grid((unsigned)((n + 255) / 256)), block(256);
    if (wbits == 8) k_block_dots_q8<8><<<grid, block, 0, st>>>(q, rows, K, xq, acc);
    else if (wbits == 4) k_block_dots_q8<4><<<grid, block, 0, st>>>(q, rows, K, xq, acc);
    else k_block_dots_q8<2><<<grid, block, 0, st>>>(q, rows, K, xq, acc);
    return cudaGetLastError();
}

}  // namespace qrx
