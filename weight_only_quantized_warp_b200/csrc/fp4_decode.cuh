// fp4_decode.cuh -- MXFP4 (e2m1) codes to bf16 for the FFN kernels.
//
// An e2m1 code is sign (bit 3), two exponent bits and one mantissa bit; its
// magnitudes by the low three bits are 0, 0.5, 1, 1.5, 2, 3, 4, 6, all exact
// in bf16: 0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0.
// The high and the low byte of those bf16 values form two 8-entry byte
// tables, looked up with byte permutes (the selector nibbles are the
// magnitude indices); the sign bit moves to bit 15 of its half.
#pragma once

#include <cstdint>

namespace qmoe {

// Two codes: the one in bits 0-3 of t to the low bf16 half, the one in bits
// 16-19 to the high half.
__device__ __forceinline__ uint32_t fp4x2_to_bf16x2(uint32_t t) {
    const uint32_t idx = t & 0x00070007u;
    const uint32_t sel = idx | (idx >> 8);                               // nibble 0: low, nibble 2: high index
    const uint32_t lo = __byte_perm(0xC0800000u, 0xC0804000u, sel);       // low bytes -> bytes 0 and 2
    const uint32_t hi = __byte_perm(0x3F3F3F00u, 0x40404040u, sel << 4);  // high bytes -> bytes 1 and 3
    return lo | hi | ((t << 12) & 0x80008000u);
}

// Eight codes of one packed word in the register order of the int4 decode:
// A[i] holds the codes in nibbles i (low half) and i + 4 (high half).
__device__ __forceinline__ void decode_fp4x8(uint32_t w, uint32_t (&A)[4]) {
    A[0] = fp4x2_to_bf16x2(w);
    A[1] = fp4x2_to_bf16x2(w >> 4);
    A[2] = fp4x2_to_bf16x2(w >> 8);
    A[3] = fp4x2_to_bf16x2(w >> 12);
}

// One code (the low four bits of c) as a float.
__device__ __forceinline__ float fp4_to_float(uint32_t c) {
    return __uint_as_float(fp4x2_to_bf16x2(c & 0xFu) << 16);
}

}  // namespace qmoe
