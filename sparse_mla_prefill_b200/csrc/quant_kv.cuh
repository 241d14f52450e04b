// Quantized latent rows: the formats, the quantize kernel and the dequantizing loads the
// attention producers use.
//
// The pages run their full model on a quantized KV cache ("Q4_0 K/V cache", "Q8 K / Q4
// V": "perf(ds4): extend sparse prefill scheduling to 10K", Production workflow and the
// clean-head validation) without defining the formats. This library reads them as block
// formats of 32 values, each block with one fp16 scale d:
//   Q8_0  codes q in [-127, 127], value d*q;     d = max|x| / 127
//   Q4_0  codes n in [0, 15],     value d*(n-8); d = m / -8, m the block's first value
//         of largest magnitude
// Codes are decided in fp32: x / d (IEEE division) rounded half to even, clamped.
// A stored row is its codes (Q8_0: one byte each; Q4_0: byte b of a block holds value b
// in the low nibble and value b+16 in the high nibble), then the row's fp16 scales,
// then zeros up to a multiple of 16 bytes. One latent row is both key (576 values) and
// value (its first 512), so a quantized cache stores each row once.
#pragma once

#include <cuda_fp16.h>

#include "device_common.cuh"

namespace ds4sp {

constexpr int kQBlock = 32;
// kFmtQ8Q4 ("Q8 K / Q4 V"): keys and values at different precisions. A stored row is the
// Q8_0 row of all the latent values (the key) followed by the Q4_0 row of the first 512
// (the value).
constexpr int kFmtF16 = 0, kFmtQ8 = 1, kFmtQ4 = 2, kFmtQ8Q4 = 3;
constexpr int kValueDims = 512;

__host__ __device__ constexpr int quant_code_bytes(int fmt, int dims) {
    return fmt == kFmtQ8 ? dims : dims / 2;
}
__host__ __device__ constexpr int quant_row_bytes(int fmt, int dims) {
    return fmt == kFmtQ8Q4 ? quant_row_bytes(kFmtQ8, dims) + quant_row_bytes(kFmtQ4, kValueDims)
                           : (quant_code_bytes(fmt, dims) + 2 * (dims / kQBlock) + 15) / 16 * 16;
}

// One thread per (row, block): quantize 32 fp16 values of row r (values dims, stride
// x_ld) in format fmt (Q8_0 or Q4_0) into the part of an output row of out_ld bytes that
// starts at byte out_off: codes, fp16 scales, zero padding to a multiple of 16 bytes.
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const __half* __restrict__ x, int x_ld, int rows, int dims, int fmt,
                     uint8_t* __restrict__ out, int out_ld, int out_off) {
    const int nb = dims / kQBlock;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)rows * nb) return;
    const int r = (int)(gid / nb), b = (int)(gid % nb);
    const __half* src = x + (size_t)r * x_ld + b * kQBlock;
    const int rb = quant_row_bytes(fmt, dims), cb = quant_code_bytes(fmt, dims);
    uint8_t* row = out + (size_t)r * out_ld + out_off;
    float v[kQBlock];
#pragma unroll
    for (int i = 0; i < kQBlock; ++i) v[i] = __half2float(src[i]);
    __half d16;
    if (fmt == kFmtQ8) {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kQBlock; ++i) amax = fmaxf(amax, fabsf(v[i]));
        d16 = __float2half_rn(amax / 127.f);               // >= +0
        const float d = __half2float(d16);
#pragma unroll
        for (int i = 0; i < kQBlock; ++i) {
            const float q = d == 0.f ? 0.f : fminf(fmaxf(rintf(v[i] / d), -127.f), 127.f);
            row[b * kQBlock + i] = (uint8_t)(int8_t)(int)q;
        }
    } else {
        float m = v[0], am = fabsf(v[0]);
#pragma unroll
        for (int i = 1; i < kQBlock; ++i)
            if (fabsf(v[i]) > am) {                 // strict: the first extreme wins
                am = fabsf(v[i]);
                m = v[i];
            }
        d16 = __float2half_rn(m / -8.f);
        if (__half2float(d16) == 0.f) d16 = __float2half_rn(0.f);   // +0 for an all-zero block
        const float d = __half2float(d16);
        uint8_t n[kQBlock];
#pragma unroll
        for (int i = 0; i < kQBlock; ++i)
            n[i] = d == 0.f ? 8 : (uint8_t)(int)fminf(fmaxf(rintf(v[i] / d) + 8.f, 0.f), 15.f);
#pragma unroll
        for (int i = 0; i < kQBlock / 2; ++i) row[b * 16 + i] = (uint8_t)(n[i] | (n[i + 16] << 4));
    }
    const unsigned short bits = __half_as_ushort(d16);
    row[cb + 2 * b] = (uint8_t)(bits & 0xff);
    row[cb + 2 * b + 1] = (uint8_t)(bits >> 8);
    if (b == 0)
        for (int i = cb + 2 * nb; i < rb; ++i) row[i] = 0;
}

// ---------------------------------------------------------------- dequantizing loads

// (1024 + u) as fp16 for two bytes picked by `sel` from `w` (bytes 0-3) and 0x64 bytes.
__device__ __forceinline__ __half2 biased_pair(uint32_t w, uint32_t sel) {
    const uint32_t h = __byte_perm(w, 0x64646464u, sel);
    return *reinterpret_cast<const __half2*>(&h);
}

// Eight fp16 values of one 16-byte chunk in the attention ring: d*q (Q8_0), q from the
// bytes of two words (lo: values 0-3, hi: values 4-7). (1024 + (q+128)) - 1152 = q is
// exact in fp16, and the product by d is rounded once.
__device__ __forceinline__ uint4 dequant_q8_chunk(uint32_t lo, uint32_t hi, __half2 d2) {
    const __half2 off = __float2half2_rn(1152.f);
    lo ^= 0x80808080u;
    hi ^= 0x80808080u;
    uint4 r;
    __half2 t;
    t = __hmul2(__hsub2(biased_pair(lo, 0x5140), off), d2); r.x = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(lo, 0x7362), off), d2); r.y = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(hi, 0x5140), off), d2); r.z = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(hi, 0x7362), off), d2); r.w = *reinterpret_cast<uint32_t*>(&t);
    return r;
}

// Eight fp16 values d*(n-8) (Q4_0) from the nibbles of two words already masked to one
// nibble per byte (w0: values 0-3, w1: values 4-7).
__device__ __forceinline__ uint4 dequant_q4_chunk(uint32_t w0, uint32_t w1, __half2 d2) {
    const __half2 off = __float2half2_rn(1032.f);
    uint4 r;
    __half2 t;
    t = __hmul2(__hsub2(biased_pair(w0, 0x5140), off), d2); r.x = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(w0, 0x7362), off), d2); r.y = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(w1, 0x5140), off), d2); r.z = *reinterpret_cast<uint32_t*>(&t);
    t = __hmul2(__hsub2(biased_pair(w1, 0x7362), off), d2); r.w = *reinterpret_cast<uint32_t*>(&t);
    return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace ds4sp
