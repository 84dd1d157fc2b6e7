// The packed int4 key codes as floats, shared by the KV4 consumer kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qkq {

// 8 codes of one 32-bit word (channel 8j + e in nibble e, two's complement) as 4 float
// pairs (channels 2k, 2k + 1).
__device__ __forceinline__ void codes_to_float2(uint32_t w, float2 (&c)[4])
{
    const uint32_t wb = w ^ 0x88888888u;  // nibble = code + 8
    const uint32_t ev = wb & 0x0F0F0F0Fu, od = (wb >> 4) & 0x0F0F0F0Fu;
    const float2 bias = make_float2(-8388616.0f, -8388616.0f);  // 2^23 + 8, exact
#pragma unroll
    for (int k = 0; k < 4; ++k)
        c[k] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u | k)),
                                      __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u | k))),
                          bias);
}

// The same 8 codes as 4 bf16 pairs (channels 2k, 2k + 1 in the low and high halves), exact:
// a nibble n = code + 8 becomes the bf16 of 128 + n (bits 0x4300 | n: 128 has an ulp of 1 in
// bf16), then 136 is subtracted in bf16 (small integers: exact).
__device__ __forceinline__ void codes_to_bf16x2(uint32_t w, uint32_t (&c)[4])
{
    const uint32_t wb = w ^ 0x88888888u;  // nibble = code + 8
    const uint32_t ev = wb & 0x0F0F0F0Fu, od = (wb >> 4) & 0x0F0F0F0Fu;
    const __nv_bfloat162 bias = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // bytes (even k, even k, odd k, odd k), then 0x43 in bytes 1 and 3
        const uint32_t x = __byte_perm(ev, od, static_cast<uint32_t>(k | (k << 4) | ((4 + k) << 8) | ((4 + k) << 12)));
        const uint32_t y = (x & 0x00FF00FFu) | 0x43004300u;
        const __nv_bfloat162 v = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&y), bias);
        c[k] = *reinterpret_cast<const uint32_t *>(&v);
    }
}

}  // namespace qkq
