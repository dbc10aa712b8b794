// qrx_dev.cuh -- device helpers shared by the qrx CUDA kernels (sm_100a).
//
// Packed weight formats (README "JustVugg/colibri", section "已实现的功能":
// int8 / packed int4 / packed int2, per-row scale, dequantised on use; the
// packed values are bit-consistent with the int8 container):
//   int8: one two's-complement code per byte;
//   int4: two codes per byte, element 2i in bits [3:0], 2i+1 in bits [7:4];
//   int2: four codes per byte, element 4i in bits [1:0] ... 4i+3 in [7:6].
//
// A "chunk" is the 16 bytes one lane loads at a time: 16 (int8), 32 (int4)
// or 64 (int2) consecutive codes of one row.  Unpacking turns the chunk's 4
// words into byte vectors that __dp4a can take; int4 and int2 fields are
// flipped to offset binary (code + 8, code + 2, all in [0, 15]) so no sign
// extension is needed; the offset is removed once per block through the sum
// of the activation digits (acc starts at -offset * sum(digits)).
//
// Activations enter the integer dot as "digit planes": per 32-element block a
// power-of-two (f32 / bf16 inputs) or Q8_0 (amax/127) scale sigma_b, and NDIG
// signed 8-bit digits per element with x ~= sigma_b * (d0 + 256 d1 + 65536 d2).
//   NDIG = 1: Q8_0 codes (README: Q8_0-style int8 activations), exact;
//   NDIG = 3: f32 or bf16 inputs held as a 22-bit fixed point per block
//             (relative error <= 2^-22 of the block's largest magnitude).
// Every dot of codes by digits is an exact int32; blocks combine in f32.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace qrx {

// chunk geometry per weight format
template <int WB> struct Fmt;
template <> struct Fmt<8> {
    static constexpr int EPC = 16;     // elements per 16-byte chunk
    static constexpr int UPW = 1;      // unpacked byte-vectors per 32-bit word
    static constexpr int DW = 4;       // digit words per plane per chunk
    static constexpr int OFF = 0;      // offset added by the unpack
};
template <> struct Fmt<4> {
    static constexpr int EPC = 32, UPW = 2, DW = 8, OFF = 8;
};
template <> struct Fmt<2> {
    static constexpr int EPC = 64, UPW = 4, DW = 16, OFF = 2;
};

// Unpack word w (part of a chunk) into UPW byte vectors (offset binary for
// int4/int2).  Element order of the vectors matches digit_slot() below.
template <int WB>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&u)[Fmt<WB>::UPW])
{
    if constexpr (WB == 8) {
        u[0] = w;
    } else if constexpr (WB == 4) {
        uint32_t o = w ^ 0x88888888u;
        u[0] = o & 0x0F0F0F0Fu;          // elements 0, 2, 4, 6 of the word
        u[1] = (o >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
    } else {
        uint32_t o = w ^ 0xAAAAAAAAu;
#pragma unroll
        for (int j = 0; j < 4; ++j) u[j] = (o >> (2 * j)) & 0x03030303u;  // elements j, 4+j, 8+j, 12+j
    }
}

// Where element l (0 <= l < EPC) of a chunk sits among the chunk's digit
// words: word index and byte lane.
template <int WB>
__device__ __forceinline__ void digit_slot(int l, int &word, int &byte)
{
    if constexpr (WB == 8) {
        word = l >> 2;
        byte = l & 3;
    } else if constexpr (WB == 4) {
        int i = l >> 3, m = l & 7;
        word = 2 * i + (m & 1);
        byte = m >> 1;
    } else {
        int i = l >> 4, m = l & 15;
        word = 4 * i + (m & 3);
        byte = m >> 2;
    }
}

// Element (within its chunk) held in byte b of unpacked vector j of chunk word i:
// the inverse of digit_slot().
template <int WB>
__device__ __forceinline__ int elem_in_chunk(int i, int j, int b)
{
    if constexpr (WB == 8) return 4 * i + b;
    else if constexpr (WB == 4) return 8 * i + 2 * b + j;
    else return 16 * i + 4 * b + j;
}

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c)
{
    return __dp4a((int)a, (int)b, c);
}

// 16-byte streaming load of weights (read once: do not keep in L1).
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Split an integer |v| < 2^22 into balanced signed bytes d0 + 256 d1 + 65536 d2.
__device__ __forceinline__ void split3(int v, int8_t &d0, int8_t &d1, int8_t &d2)
{
    int a = (int)(int8_t)(v & 0xFF);
    int r = (v - a) >> 8;
    int b = (int)(int8_t)(r & 0xFF);
    int c = (r - b) >> 8;
    d0 = (int8_t)a;
    d1 = (int8_t)b;
    d2 = (int8_t)c;
}

// Exponent shift s of the 22-bit fixed point of a block with largest magnitude
// amax > 0: amax * 2^s lies in [2^21, 2^22), so rint(x * 2^s) fits split3 and
// the block scale is sigma = 2^-s.
__device__ __forceinline__ int fixed_shift(float amax)
{
    int e;
    frexpf(amax, &e);     // amax = f * 2^e with f in [0.5, 1)
    return 22 - e;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Q8_0 code of x given f = 127/amax: round-half-away of the f32 product,
// clamped to [-127, 127] on the product (an infinite f from a tiny amax still
// gives +-127; 0 * inf gives 0).
__device__ __forceinline__ int q8_code(float x, float f)
{
    const float v = __fmul_rn(x, f);
    if (v != v) return 0;
    if (v >= 127.f) return 127;
    if (v <= -127.f) return -127;
    return (int)roundf(v);
}

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g / (1.0f + expf(-g)) * u;
}

// Programmatic dependent launch.  pdl_wait() blocks until the previous kernel
// in the stream has completed and its memory is visible (a no-op when the
// kernel was launched without the programmatic-serialization attribute);
// pdl_trigger() lets the next kernel begin launching.  Every kernel triggers
// only after its own wait, so a kernel that starts early can rely on all
// kernels before its predecessor having completed.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Device-side sticky status flag (set by kernels, read by qrx_last_error).
// The library is built as one translation unit, so there is one flag per device.
enum { DERR_NONE = 0, DERR_BOUNDS = 1, DERR_TIMEOUT = 2, DERR_BADIDX = 3 };
__device__ int g_status;

__device__ __forceinline__ void raise_status(int code)
{
    atomicCAS(&g_status, 0, code);
}

// Adaptive expert top-p for one token, run by a whole warp (README
// "JustVugg/colibri", section "快速开始": the --topp knob).  Lane j < k holds
// the weight wv of slot j.  Slots are taken by weight, largest first (equal
// weights: the lower slot first), their weights summed in double in that
// order, until the sum reaches thr = p * rsf; returns whether this lane's slot
// was taken (lanes >= k: false).  Every lane runs the same steps.
__device__ __forceinline__ bool warp_topp_keep(int lane, int k, float wv, double thr)
{
    bool taken = false;
    double c = 0.0;
    for (int n = 0; n < k; ++n) {
        float best = (lane < k && !taken) ? wv : 0.f;
        int bj = (lane < k && !taken) ? lane : 0x7fffffff;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            const bool better = oj != 0x7fffffff && (bj == 0x7fffffff || ob > best || (ob == best && oj < bj));
            if (better) { best = ob; bj = oj; }
        }
        if (lane == bj) taken = true;
        c += (double)best;
        if (c >= thr) break;
    }
    return taken;
}

}  // namespace qrx
