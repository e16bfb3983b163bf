// io16.cuh -- the 16-bit I/O element types of the tensor-core paths: bfloat16 and
// float16 (the page's section "Implementacion" lists FP32 and FP16 kernels; bf16 is the
// tensor-core type of the workloads here).  Per type: unpacking the halves of a 32-bit
// word to fp32, packing two fp32 values (round to nearest even), and the operand format
// code of the tcgen05 instruction descriptor (kind::f16: 0 = F16, 1 = BF16; A and B
// always share one type).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace eqlin {

template <class T>
struct Io16;

template <>
struct Io16<__nv_bfloat16> {
    static constexpr uint32_t kUmmaFormat = 1;
    __device__ __forceinline__ static float lo(uint32_t w) { return __uint_as_float(w << 16); }
    __device__ __forceinline__ static float hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
    __device__ __forceinline__ static uint32_t pack(float a, float b) {
        __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __host__ __device__ static __nv_bfloat16 from_float(float v) { return __float2bfloat16_rn(v); }
};

template <>
struct Io16<__half> {
    static constexpr uint32_t kUmmaFormat = 0;
    __device__ __forceinline__ static float lo(uint32_t w) {
        return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
    }
    __device__ __forceinline__ static float hi(uint32_t w) {
        return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
    }
    __device__ __forceinline__ static uint32_t pack(float a, float b) {
        __half2 v = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __host__ __device__ static __half from_float(float v) { return __float2half_rn(v); }
};

}  // namespace eqlin
