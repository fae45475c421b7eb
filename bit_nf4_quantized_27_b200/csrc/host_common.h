// Host-side helpers of the C ABI: device checks, argument validation, tables.
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "qlora_nf4.h"

namespace qlora {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Current device must be an sm_100 part; cached per device ordinal.
inline qlora_status check_device(int *dev_out, int *sm_count) {
  static std::mutex mu;
  static int cached_major[64];
  static int cached_sms[64];
  static bool known[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= 64) return QLORA_ERR_NO_DEVICE;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!known[dev]) {
      int major = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return QLORA_ERR_NO_DEVICE;
      }
      cached_major[dev] = major;
      cached_sms[dev] = sms;
      known[dev] = true;
    }
    if (cached_major[dev] != 10) return QLORA_ERR_NO_DEVICE;
    if (dev_out) *dev_out = dev;
    if (sm_count) *sm_count = cached_sms[dev];
  }
  return QLORA_OK;
}

inline qlora_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

inline qlora_status check_nf4(const qlora_nf4_tensor *t) {
  if (!t || !t->codes || !t->scale_codes || !t->c2) return QLORA_ERR_INVALID_ARGUMENT;
  if (t->rows <= 0 || t->cols <= 0 || t->cols % QLORA_BLOCK) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (t->rows > (int64_t(1) << 31) || t->cols > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(t->codes, 16) || !aligned(t->c2, 4)) return QLORA_ERR_MISALIGNED;
  if (t->scale_format < QLORA_SCALE_E4M3 || t->scale_format > QLORA_SCALE_U8) return QLORA_ERR_INVALID_ARGUMENT;
  return QLORA_OK;
}

// ---------------------------------------------------------------------------
// Float32 code search table (see quant_kernels.cuh).  Built from the plain float32
// definition of the code: argmin_j |x - L_j|, lowest j on ties.
// ---------------------------------------------------------------------------
inline uint32_t f32_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
inline float bits_f32(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
// Monotone map float32 -> uint32 (for bisection over the ordered float line).
inline uint32_t f32_key(float f) { uint32_t u = f32_bits(f); return (u & 0x80000000u) ? ~u : (u | 0x80000000u); }
inline float key_f32(uint32_t k) { return bits_f32((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

inline const float *nf4_levels_host() {
  static float lv[16];
  static std::once_flag once;
  static const uint32_t bits[16] = {0xbf800000u, 0xbf3239b3u, 0xbf066b30u, 0xbeca32a0u, 0xbe91a24cu, 0xbe3d353fu,
                                    0xbdba786bu, 0x00000000u, 0x3da2fb03u, 0x3e24cae1u, 0x3e7c04dcu, 0x3ead0338u,
                                    0x3ee1a4b7u, 0x3f1007aau, 0x3f3913b1u, 0x3f800000u};
  std::call_once(once, [] { for (int i = 0; i < 16; ++i) lv[i] = bits_f32(bits[i]); });
  return lv;
}

inline int code_of(float x) {
  const float *L = nf4_levels_host();
  volatile float best = std::fabs(x - L[0]);  // volatile: float32 rounding, no contraction
  int bi = 0;
  for (int j = 1; j < 16; ++j) {
    volatile float d = std::fabs(x - L[j]);
    if (d < best) { best = d; bi = j; }
  }
  return bi;
}

// Cell of x: round-to-nearest of x*32 + 32, read from the low mantissa bits of
// fl32(x*32 + 32 + 1.5*2^23) (one fused multiply-add, exact integer spacing
// there); 0..64 for x in [-1, 1].
constexpr float kCellMagic = 12582912.0f + 32.0f;  // 1.5 * 2^23 + 32
inline int cell_of(float x) {
  const float v = std::fmaf(x, 32.0f, kCellMagic);
  return static_cast<int>(v - 12582912.0f);
}

struct HostCellTable {
  float thr[65];
  uint32_t base[65];
  float switch_points[15];
  uint32_t min_edge_ulps;  // fewest float32 steps between a switch point and a cell edge
  bool ok;
};

inline const HostCellTable &cell_table() {
  static HostCellTable t;
  static std::once_flag once;
  std::call_once(once, [] {
    const float *L = nf4_levels_host();
    t.ok = true;
    // Switch points: t_j = largest x with code(x) <= j, by bisection on the float line.
    for (int j = 0; j < 15; ++j) {
      uint32_t lo = f32_key(L[j]), hi = f32_key(L[j + 1]);  // code(lo) = j, code(hi) = j+1
      while (hi - lo > 1) {
        const uint32_t mid = lo + (hi - lo) / 2;
        if (code_of(key_f32(mid)) <= j) lo = mid; else hi = mid;
      }
      t.switch_points[j] = key_f32(lo);
    }
    // Cell k = [b_k, b_{k+1}): b_k = smallest x in [-1-2^-20, 1+2^-20] with cell(x) >= k.
    const float xmin = -1.0f - 1.0f / (1 << 20), xmax = 1.0f + 1.0f / (1 << 20);
    float b[67];
    for (int k = 0; k <= 66; ++k) {
      uint32_t lo = f32_key(xmin), hi = f32_key(xmax);
      if (cell_of(key_f32(lo)) >= k) { b[k] = key_f32(lo); continue; }
      if (cell_of(key_f32(hi)) < k) { b[k] = xmax; continue; }
      while (hi - lo > 1) {
        const uint32_t mid = lo + (hi - lo) / 2;
        if (cell_of(key_f32(mid)) >= k) hi = mid; else lo = mid;
      }
      b[k] = key_f32(hi);
    }
    // The kernel picks the cell from x' = fl32(w * r), r an approximate
    // reciprocal of S, within 6 ulp of fl32(w / S), and checks only the chosen
    // cell's switch point for an 8-ulp band: that is exact only while no switch
    // point lies within 6 ulp of a cell edge, where x' and the exact quotient
    // could fall into different cells.  Keep every switch point more than
    // kEdgeUlps float32 steps from every edge.
    constexpr uint32_t kEdgeUlps = 8;
    t.min_edge_ulps = 0xffffffffu;
    for (int j = 0; j < 15; ++j)
      for (int k = 0; k <= 66; ++k) {
        const uint32_t a = f32_key(t.switch_points[j]), e = f32_key(b[k]);
        const uint32_t d = a > e ? a - e : e - a;
        if (d < t.min_edge_ulps) t.min_edge_ulps = d;
      }
    if (t.min_edge_ulps <= kEdgeUlps) t.ok = false;
    for (int k = 0; k < 65; ++k) {
      const double lo = b[k], hi = b[k + 1];
      int inside = 0, best = 0;
      double bd = 1e30;
      for (int j = 0; j < 15; ++j) {
        const double s = t.switch_points[j];
        const double d = s < lo ? lo - s : (s >= hi ? s - hi : 0.0);
        if (d == 0.0) ++inside;
        if (d < bd) { bd = d; best = j; }
      }
      if (inside > 1) t.ok = false;
      t.thr[k] = t.switch_points[best];
      t.base[k] = static_cast<uint32_t>(best);
    }
    // Self-check the table against the definition at both ends of every cell and
    // around every switch point.
    for (int k = 0; k < 65 && t.ok; ++k) {
      const float ends[2] = {b[k], std::nextafter(b[k + 1], -2.0f)};
      for (float x : ends) {
        if (x < -1.0f || x > 1.0f) continue;
        const int c = cell_of(x);
        if (static_cast<int>(t.base[c] + (x > t.thr[c] ? 1 : 0)) != code_of(x)) t.ok = false;
      }
    }
    for (int j = 0; j < 15 && t.ok; ++j) {
      float x = t.switch_points[j];
      for (int s = 0; s < 8; ++s) x = std::nextafter(x, -2.0f);
      for (int s = 0; s < 17; ++s, x = std::nextafter(x, 2.0f)) {
        const int c = cell_of(x);
        if (static_cast<int>(t.base[c] + (x > t.thr[c] ? 1 : 0)) != code_of(x)) t.ok = false;
      }
    }
  });
  return t;
}

}  // namespace qlora
