// The packed int4 key codes as floats, shared by the KV4 consumer kernels.
#pragma once

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

}  // namespace qkq
