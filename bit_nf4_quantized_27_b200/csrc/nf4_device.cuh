// Device-side helpers shared by the NF4 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qlora_nf4.h"

namespace qlora {

constexpr int kBlock = QLORA_BLOCK;  // weights per absmax block
constexpr int kGroup = QLORA_GROUP;  // blocks per second-level group

// The 16 NF4 levels as float32 bit patterns: Phi^-1 at the quantile offsets of the
// QLoRA glossary page's snippet ("How QLoRA works"; offset 0.9677083, 8 positive and
// 7 negative quantiles plus an exact zero, sorted, divided by the largest), each
// evaluated in exact arithmetic and rounded once to float32.
__constant__ uint32_t kNf4LevelBits[16] = {
    0xbf800000u, 0xbf3239b3u, 0xbf066b30u, 0xbeca32a0u, 0xbe91a24cu, 0xbe3d353fu,
    0xbdba786bu, 0x00000000u, 0x3da2fb03u, 0x3e24cae1u, 0x3e7c04dcu, 0x3ead0338u,
    0x3ee1a4b7u, 0x3f1007aau, 0x3f3913b1u, 0x3f800000u};

// The same 16 levels as compile-time float constants (identical bit patterns;
// a CPU test checks the two lists against each other), so that kernels can use
// them as instruction immediates instead of registers.  j must be a constant
// after unrolling.
__host__ __device__ constexpr float nf4_level(int j) {
  return j == 0 ? -0x1.000000p+0f : j == 1 ? -0x1.647366p-1f : j == 2 ? -0x1.0cd660p-1f
       : j == 3 ? -0x1.946540p-2f : j == 4 ? -0x1.234498p-2f : j == 5 ? -0x1.7a6a7ep-3f
       : j == 6 ? -0x1.74f0d6p-4f : j == 7 ? 0x0.0p+0f : j == 8 ? 0x1.45f606p-4f
       : j == 9 ? 0x1.4995c2p-3f : j == 10 ? 0x1.f809b8p-3f : j == 11 ? 0x1.5a0670p-2f
       : j == 12 ? 0x1.c3496ep-2f : j == 13 ? 0x1.200f54p-1f : j == 14 ? 0x1.722762p-1f
       : 0x1.000000p+0f;
}

// Device status word flags (bit k set <=> status code k was raised).
__device__ __forceinline__ void raise_status(uint32_t *status, qlora_status code) {
  if (status) atomicOr(status, 1u << static_cast<uint32_t>(code));
}

// Scale-code formats of the second level (qlora_scale_format): 0 OCP FP8 E4M3,
// 1 OCP FP8 E5M2, 2 linear unsigned byte.  The group maximum maps to the
// format's largest value.
__host__ __device__ constexpr float scale_format_max(int fmt) {
  return fmt == 1 ? 57344.0f : fmt == 2 ? 255.0f : 448.0f;
}

// E4M3 byte -> float32 (exact: every E4M3 value is a half value).
__device__ __forceinline__ float e4m3_to_f32(uint8_t q) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3);
  return __half2float(__half(h));
}

// float32 -> E4M3 byte, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// Exact float32 value of a scale code in format fmt (E4M3 and E5M2 values are
// half values; a byte is an integer).
__device__ __forceinline__ float scale_code_value(uint32_t q, int fmt) {
  if (fmt == 2) return static_cast<float>(q & 0xffu);
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q & 0xffu),
                                               fmt == 1 ? __NV_E5M2 : __NV_E4M3);
  return __half2float(__half(h));
}
// The values of the two scale codes in the low 16 bits of q (low byte first).
__device__ __forceinline__ float2 scale_code_value2(uint32_t q, int fmt) {
  if (fmt == 2) return make_float2(static_cast<float>(q & 0xffu), static_cast<float>((q >> 8) & 0xffu));
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(q & 0xffffu),
                                                   fmt == 1 ? __NV_E5M2 : __NV_E4M3);
  return __half22float2(__half2(h));
}
// Scale code of a non-negative float32 in format fmt: round to nearest even,
// saturating at the format's largest value.
__device__ __forceinline__ uint8_t scale_code_encode(float x, int fmt) {
  if (fmt == 2) return static_cast<uint8_t>(min(__float2uint_rn(x), 255u));
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, fmt == 1 ? __NV_E5M2 : __NV_E4M3));
}

// Two float32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Dequantised block scale S' = fl32(E4M3(q) * c2).
__device__ __forceinline__ float block_scale(const uint8_t *scale_codes, const float *c2, int64_t b, int fmt) {
  return __fmul_rn(scale_code_value(__ldg(scale_codes + b), fmt), __ldg(c2 + (b >> 8)));
}

}  // namespace qlora
