// Device helpers shared by the tcgen05 forward and backward kernels:
// bf16 loads from the input ring and the compensated (hi + lo) bf16 operand
// writer for MN-major B operands.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace m2rnn {

// Loads n bf16 values (n = 4 or a multiple of 8; 8- or 16-byte aligned) from shared memory.
template <int N>
__device__ __forceinline__ void lds_bf16(const uint16_t* src, float (&out)[N]) {
    if constexpr (N % 8 == 0) {
#pragma unroll
        for (int g = 0; g < N / 8; ++g) {
            const uint4 w = *reinterpret_cast<const uint4*>(src + 8 * g);
            out[8 * g + 0] = bf16lo_to_f32(w.x); out[8 * g + 1] = bf16hi_to_f32(w.x);
            out[8 * g + 2] = bf16lo_to_f32(w.y); out[8 * g + 3] = bf16hi_to_f32(w.y);
            out[8 * g + 4] = bf16lo_to_f32(w.z); out[8 * g + 5] = bf16hi_to_f32(w.z);
            out[8 * g + 6] = bf16lo_to_f32(w.w); out[8 * g + 7] = bf16hi_to_f32(w.w);
        }
    } else {
        static_assert(N == 4, "lds_bf16");
        const uint2 w = *reinterpret_cast<const uint2*>(src);
        out[0] = bf16lo_to_f32(w.x); out[1] = bf16hi_to_f32(w.x);
        out[2] = bf16lo_to_f32(w.y); out[3] = bf16hi_to_f32(w.y);
    }
}

// hi / lo bf16 pair of two fp32 values, packed two per 32-bit word
// (element with the lower index in the low half).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
    hi = __byte_perm(b0, b1, 0x7632);
    const float l0 = x0 - __uint_as_float(b0 & 0xFFFF0000u);
    const float l1 = x1 - __uint_as_float(b1 & 0xFFFF0000u);
    const __nv_bfloat162 lp = __floats2bfloat162_rn(l0, l1);
    lo = *reinterpret_cast<const uint32_t*>(&lp);
}

// Same pair with the hi part rounded to nearest (unbiased): used where the
// hi part alone feeds a product (the dW MMA of the backward).
__device__ __forceinline__ void split_pack_rn(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
    hi = *reinterpret_cast<const uint32_t*>(&hp);
    const float l0 = x0 - bf16lo_to_f32(hi);
    const float l1 = x1 - bf16hi_to_f32(hi);
    const __nv_bfloat162 lp = __floats2bfloat162_rn(l0, l1);
    lo = *reinterpret_cast<const uint32_t*>(&lp);
}

// Writes this thread's RT state values of column j into the MN-major B
// operand of its tile: element (k = j, n) lives at
//   (j/8)·(NT·16) + (n/8)·128 + (j%8)·16 + (n%8)·2,
// hi values at n = nloc + r, lo values at n = R + nloc + r.
template <class C, bool RN = false>
__device__ __forceinline__ void write_state_operand(uint8_t* Bt, const float (&h)[C::RT], int j, int nloc) {
    auto split = [](float a, float b, uint32_t& hi, uint32_t& lo) {
        if constexpr (RN) split_pack_rn(a, b, hi, lo);
        else split_pack(a, b, hi, lo);
    };
    uint8_t* colbase = Bt + (j >> 3) * (C::NT * 16) + (j & 7) * 16;
    if constexpr (C::RT % 8 == 0) {
#pragma unroll
        for (int g = 0; g < C::RT / 8; ++g) {
            uint4 hi, lo;
            split(h[8 * g + 0], h[8 * g + 1], hi.x, lo.x);
            split(h[8 * g + 2], h[8 * g + 3], hi.y, lo.y);
            split(h[8 * g + 4], h[8 * g + 5], hi.z, lo.z);
            split(h[8 * g + 6], h[8 * g + 7], hi.w, lo.w);
            const int n = nloc + 8 * g;
            *reinterpret_cast<uint4*>(colbase + (n >> 3) * 128) = hi;
            *reinterpret_cast<uint4*>(colbase + ((C::R + n) >> 3) * 128) = lo;
        }
    } else {
        uint2 hi, lo;
        split(h[0], h[1], hi.x, lo.x);
        split(h[2], h[3], hi.y, lo.y);
        const int n = nloc;
        *reinterpret_cast<uint2*>(colbase + (n >> 3) * 128 + (n & 7) * 2) = hi;
        *reinterpret_cast<uint2*>(colbase + ((C::R + n) >> 3) * 128 + ((C::R + n) & 7) * 2) = lo;
    }
}

// Writes only the hi parts (bf16, round to nearest) of this thread's RT
// values of column j, at n = nloc + r: for operands whose lo half no MMA reads.
// NB: rows of the buffer (the same layout with NB in place of NT).
template <class C, int NB = C::NT>
__device__ __forceinline__ void write_state_operand_hi(uint8_t* Bt, const float (&h)[C::RT], int j, int nloc) {
    uint8_t* colbase = Bt + (j >> 3) * (NB * 16) + (j & 7) * 16;
    auto pack = [](float a, float b) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&v);
    };
    if constexpr (C::RT % 8 == 0) {
#pragma unroll
        for (int g = 0; g < C::RT / 8; ++g) {
            const uint4 hi = make_uint4(pack(h[8 * g], h[8 * g + 1]), pack(h[8 * g + 2], h[8 * g + 3]),
                                        pack(h[8 * g + 4], h[8 * g + 5]), pack(h[8 * g + 6], h[8 * g + 7]));
            *reinterpret_cast<uint4*>(colbase + ((nloc + 8 * g) >> 3) * 128) = hi;
        }
    } else {
        const uint2 hi = make_uint2(pack(h[0], h[1]), pack(h[2], h[3]));
        *reinterpret_cast<uint2*>(colbase + (nloc >> 3) * 128 + (nloc & 7) * 2) = hi;
    }
}

// The bf16 state values (round to nearest) of one thread's RT rows of its
// column in a state operand, at the thread's own position tp within it:
// tp = operand + (j/8)·(R·16) + (j%8)·16 + (nloc/8)·128 + (nloc%8)·2, the
// layout of write_state_operand_hi<C, R> (the next 8-row group 128 bytes on).
template <class C>
__device__ __forceinline__ void put_state_hi(uint8_t* tp, const float (&h)[C::RT]) {
    auto pack = [](float a, float b) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&v);
    };
    if constexpr (C::RT % 8 == 0) {
#pragma unroll
        for (int g = 0; g < C::RT / 8; ++g)
            *reinterpret_cast<uint4*>(tp + g * 128) =
                make_uint4(pack(h[8 * g], h[8 * g + 1]), pack(h[8 * g + 2], h[8 * g + 3]),
                           pack(h[8 * g + 4], h[8 * g + 5]), pack(h[8 * g + 6], h[8 * g + 7]));
    } else {
        *reinterpret_cast<uint2*>(tp) = make_uint2(pack(h[0], h[1]), pack(h[2], h[3]));
    }
}
template <class C>
__device__ __forceinline__ void get_state_hi(const uint8_t* tp, float (&h)[C::RT]) {
    if constexpr (C::RT % 8 == 0) {
#pragma unroll
        for (int g = 0; g < C::RT / 8; ++g) {
            const uint4 w = *reinterpret_cast<const uint4*>(tp + g * 128);
            h[8 * g + 0] = bf16lo_to_f32(w.x); h[8 * g + 1] = bf16hi_to_f32(w.x);
            h[8 * g + 2] = bf16lo_to_f32(w.y); h[8 * g + 3] = bf16hi_to_f32(w.y);
            h[8 * g + 4] = bf16lo_to_f32(w.z); h[8 * g + 5] = bf16hi_to_f32(w.z);
            h[8 * g + 6] = bf16lo_to_f32(w.w); h[8 * g + 7] = bf16hi_to_f32(w.w);
        }
    } else {
        const uint2 w = *reinterpret_cast<const uint2*>(tp);
        h[0] = bf16lo_to_f32(w.x); h[1] = bf16hi_to_f32(w.x);
        h[2] = bf16lo_to_f32(w.y); h[3] = bf16hi_to_f32(w.y);
    }
}

}  // namespace m2rnn
