// NF4 quantise (absmax per 64-block, codes, packing, E4M3 double quantisation of
// the block scales per group of 256) and dequantise kernels.
//
// Quantiser: "QLoRA" (Ultralytics glossary), "How QLoRA works": NF4 bullet (one
// absmax per 64 weights, 4-bit code into 16 normal-quantile levels) and the
// double-quantisation bullet (the block scales quantised to 8 bits in blocks of
// 256); "Grokking QLoRA" (vnread), "Double Quantization": the 8-bit format is FP8.
//
// One CTA owns one whole group (256 blocks = 16384 weights), so the group maximum
// needed by the second level is a CTA-local reduction and no scratch memory or
// second pass is needed.  Loads are 16-byte vectors; lanes 8 (bf16) or 16 (f32)
// at a time share a block and reduce its absmax with warp shuffles.
//
// Code search.  The code of x = fl32(w / S) is argmin_j fl32(|x - L_j|), lowest j
// on ties.  It is a non-decreasing step function of x with 15 switch points t_j
// (the largest float32 whose code is <= j).  The kernel cuts [-1, 1] into 65 cells
// of width 1/32, narrower than the closest pair of switch points: the cell is the
// nearest integer to x * 32 + 32, taken from the low mantissa bits of
// fl32(x * 32 + 32 + 1.5 * 2^23) (one FMA, no conversion).  It keeps per cell the
// switch point nearest to it and the code just below that point (one 8-byte
// entry): code = base + (x > thr).  The table is built on the host from the same
// float32 definition and the same cell formula; each lane reads its own copy of
// it (entry k of lane l at (32 k + l) * 8 bytes), so the lookups of a warp never
// collide in a bank.  To avoid a division per weight, the fast path uses
// x' = fl32(w * r) with r the hardware reciprocal approximation of S (absolute
// error at most 2^-23 for S in [1, 2), so relative error at most 2^-22): x' is
// within 6 ulp of fl32(w / S).  Whenever x' lies within 8 ulp of the cell's
// switch point, the exact quotient (IEEE division) is used instead, so the
// result is always the code of fl32(w / S).
#pragma once

#include "nf4_device.cuh"

namespace qlora {

constexpr int kCells = 65;

struct CodeCellTable {
  float thr[kCells];      // switch point nearest to the cell
  uint32_t base[kCells];  // code of x <= thr
};

// Cell 0..64 of x in [-1, 1] (the unsigned min keeps any other input in range).
__device__ __forceinline__ uint32_t code_cell(float x) {
  const float v = __fmaf_rn(x, 32.0f, 12582912.0f + 32.0f);
  return min(__float_as_uint(v) - 0x4B400000u, static_cast<uint32_t>(kCells - 1));
}

// Entry (switch point, base code bits) at shared address `addr`.
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// Exact code of a normalised weight x in [-1, 1] (x already equal to fl32(w / S));
// tab_lane = shared address of this lane's entry 0.
__device__ __forceinline__ uint32_t code_from_table(float x, uint32_t tab_lane) {
  const float2 e = lds_f2(tab_lane + code_cell(x) * 256u);
  return __float_as_uint(e.y) + (x > e.x ? 1u : 0u);
}

template <typename TIn>
struct QuantTraits;
template <>
struct QuantTraits<__nv_bfloat16> {
  static constexpr int kVecs = 2;           // two 16-byte vectors per lane and block
  static constexpr int kElemsPerLane = 16;
  static constexpr int kMinCtas = 4;        // resident CTAs per SM the register budget is cut for
};
template <>
struct QuantTraits<float> {
  static constexpr int kVecs = 1;
  static constexpr int kElemsPerLane = 4;
  static constexpr int kMinCtas = 1;        // sixteen 16-byte loads in flight per thread need the registers
};

// Unpacks the 16-byte vector of this lane to float32 values.
__device__ __forceinline__ void unpack_vec(const uint4 &v, float (&w)[8]) {
  w[0] = bf16lo_to_f32(v.x); w[1] = bf16hi_to_f32(v.x);
  w[2] = bf16lo_to_f32(v.y); w[3] = bf16hi_to_f32(v.y);
  w[4] = bf16lo_to_f32(v.z); w[5] = bf16hi_to_f32(v.z);
  w[6] = bf16lo_to_f32(v.w); w[7] = bf16hi_to_f32(v.w);
}
__device__ __forceinline__ void unpack_vec(const uint4 &v, float (&w)[4]) {
  w[0] = __uint_as_float(v.x); w[1] = __uint_as_float(v.y);
  w[2] = __uint_as_float(v.z); w[3] = __uint_as_float(v.w);
}

// |w| bit pattern maximum; NaN and infinities compare above every finite value.
__device__ __forceinline__ uint32_t absbits_max(const uint4 &v, __nv_bfloat16 *) {
  const uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
  const uint32_t b = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
  const uint32_t m = __vmaxu2(a, b);
  return max(m & 0xffffu, m >> 16) << 16;  // as float32 bits
}
__device__ __forceinline__ uint32_t absbits_max(const uint4 &v, float *) {
  return max(max(v.x & 0x7fffffffu, v.y & 0x7fffffffu), max(v.z & 0x7fffffffu, v.w & 0x7fffffffu));
}

constexpr int kQuantThreads = 256;

// grid.x = number of groups; one CTA per group of 256 blocks.
template <typename TIn>
__global__ void __launch_bounds__(kQuantThreads, QuantTraits<TIn>::kMinCtas)
nf4_quantize_kernel(const TIn *__restrict__ W, int64_t nblocks, uint8_t *__restrict__ codes,
                    uint8_t *__restrict__ scale_codes, float *__restrict__ c2_out,
                    uint32_t *__restrict__ status, const CodeCellTable table, int fmt) {
  constexpr int EPL = QuantTraits<TIn>::kElemsPerLane;
  constexpr int VPL = QuantTraits<TIn>::kVecs;
  constexpr int EPV = EPL / VPL;                         // elements per 16-byte vector
  constexpr int LPB = kBlock / EPL;                      // lanes per block
  constexpr int BPI = kQuantThreads / LPB;               // blocks per CTA iteration
  constexpr int ITERS = kGroup / BPI;

  __shared__ __align__(16) float2 s_tab[kCells * 32];  // (switch point, base code bits), one copy per lane
  __shared__ float s_absmax[kGroup];
  __shared__ float s_wmax[kQuantThreads / 32];

  const int tid = threadIdx.x;
  for (int e = tid; e < kCells * 32; e += kQuantThreads)
    s_tab[e] = make_float2(table.thr[e >> 5], __uint_as_float(table.base[e >> 5]));
  const uint32_t tab_lane = static_cast<uint32_t>(__cvta_generic_to_shared(s_tab)) + (tid & 31) * 8u;
  // cell k's entry from the bits of fl32(x * 32 + 32 + 1.5 * 2^23): (bits - 0x4B400000) * 256 + tab_lane,
  // one multiply-add in 32-bit arithmetic (|x'| <= 1 + 2 ulp keeps the cell in 0..64)
  const uint32_t tab_off = tab_lane - 0x4B400000u * 256u;
  uint32_t pmul[8];  // 16^i in registers the compiler cannot see through: the packing runs as multiply-adds
  {
    uint32_t m16;
    asm("mov.u32 %0, 16;" : "=r"(m16));
    pmul[0] = 1u;
#pragma unroll
    for (int i = 1; i < 8; ++i) pmul[i] = pmul[i - 1] * m16;
  }
  const int64_t g = blockIdx.x;
  const int64_t blk0 = g * kGroup;
  const int nblk = static_cast<int>(nblocks - blk0 < kGroup ? nblocks - blk0 : kGroup);

  // Issue every load of this thread first (ITERS x VPL x 16 bytes in flight).
  uint4 v[ITERS][VPL];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int lb = it * BPI + tid / LPB;  // block within group
#pragma unroll
    for (int h = 0; h < VPL; ++h) {
      if (lb < nblk) {
        const int64_t e0 = (blk0 + lb) * kBlock + (tid % LPB) * EPL + h * EPV;
        v[it][h] = __ldg(reinterpret_cast<const uint4 *>(W + e0));
      } else {
        v[it][h] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  __syncthreads();

#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int lb = it * BPI + tid / LPB;
    uint32_t mb = absbits_max(v[it][0], static_cast<TIn *>(nullptr));
#pragma unroll
    for (int h = 1; h < VPL; ++h) mb = max(mb, absbits_max(v[it][h], static_cast<TIn *>(nullptr)));
#pragma unroll
    for (int o = LPB / 2; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    if (lb >= nblk) continue;
    const bool finite = mb < 0x7f800000u;
    const float S = __uint_as_float(mb);
    if (!finite && (tid % LPB) == 0) raise_status(status, QLORA_ERR_NONFINITE);
    if ((tid % LPB) == 0) s_absmax[lb] = finite ? S : 0.0f;

    // element i of this lane's vectors, as float32 (unpacked where it is used)
    auto elem = [&](int i) -> float {
      const uint4 &q = v[it][i / EPV];
      const int j = i % EPV;
      if constexpr (EPV == 8) {
        const uint32_t wd = (j >> 1) == 0 ? q.x : (j >> 1) == 1 ? q.y : (j >> 1) == 2 ? q.z : q.w;
        return (j & 1) ? bf16hi_to_f32(wd) : bf16lo_to_f32(wd);
      } else {
        return __uint_as_float(j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w);
      }
    };
    uint64_t packed = 0;
    if (S == 0.0f || !finite) {
      packed = 0x7777777777777777ull & (EPL >= 16 ? ~0ull : ((1ull << (4 * EPL)) - 1));  // exact-zero level
    } else {
      float rS;
      asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rS) : "f"(S));
      bool slow = !(rS < 3.0e38f);  // subnormal S (flushed): every code takes the exact path
      if (slow) rS = 0.0f;          // (and the fast path's cells stay in range)
      uint32_t plo = 0, phi = 0;
      uint32_t dmin = 0xffffffffu;  // smallest (bit distance of x' from its cell's switch point) + 8
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const float xa = __fmul_rn(elem(i), rS);
        const float2 e = lds_f2(__float_as_uint(__fmaf_rn(xa, 32.0f, 12582912.0f + 32.0f)) * 256u + tab_off);
        const uint32_t c = __float_as_uint(e.y) + (xa > e.x ? 1u : 0u);
        dmin = min(dmin, __float_as_uint(xa) - __float_as_uint(e.x) + 8u);
        if (i < 8) plo = c * pmul[i & 7] + plo; else phi = c * pmul[i & 7] + phi;
      }
      slow |= dmin <= 16u;
      if (slow) {
        plo = phi = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const uint32_t c = code_from_table(__fdiv_rn(elem(i), S), tab_lane);
          if (i < 8) plo = c * pmul[i & 7] + plo; else phi = c * pmul[i & 7] + phi;
        }
      }
      packed = static_cast<uint64_t>(plo) | (static_cast<uint64_t>(phi) << 32);
    }
    const int64_t e0 = (blk0 + lb) * kBlock + (tid % LPB) * EPL;
    if constexpr (EPL == 16) {
      *reinterpret_cast<uint2 *>(codes + e0 / 2) =
          make_uint2(static_cast<uint32_t>(packed), static_cast<uint32_t>(packed >> 32));
    } else if constexpr (EPL == 8) {
      *reinterpret_cast<uint32_t *>(codes + e0 / 2) = static_cast<uint32_t>(packed);
    } else {
      *reinterpret_cast<uint16_t *>(codes + e0 / 2) = static_cast<uint16_t>(packed);
    }
  }
  __syncthreads();

  // Second level: c2 = fl32(max S / F), q = enc(fl32(S / c2)) in format fmt.
  float m = tid < nblk ? s_absmax[tid] : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) s_wmax[tid >> 5] = m;
  __syncthreads();
  m = s_wmax[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, s_wmax[i]);
  const float c2 = m == 0.0f ? 0.0f : __fdiv_rn(m, scale_format_max(fmt));
  if (tid < nblk) scale_codes[blk0 + tid] = c2 == 0.0f ? 0 : scale_code_encode(__fdiv_rn(s_absmax[tid], c2), fmt);
  if (tid == 0) c2_out[g] = c2;
}

// ---------------------------------------------------------------------------
// Dequantise: w' = bf16_rne(fl32(L[c] * S')), S' = fl32(E4M3(q) * c2).
// One thread per 16 bytes of codes (32 weights, half a block).
// ---------------------------------------------------------------------------
constexpr int kDequantThreads = 256;

template <typename TOut>
__global__ void __launch_bounds__(kDequantThreads)
nf4_dequantize_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale_codes,
                      const float *__restrict__ c2, int64_t nchunks, TOut *__restrict__ out, int fmt) {
  __shared__ float s_lv[16];
  if (threadIdx.x < 16) s_lv[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
  __syncthreads();
  for (int64_t ch = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ch < nchunks;
       ch += (int64_t)gridDim.x * blockDim.x) {
    const uint4 cv = __ldg(reinterpret_cast<const uint4 *>(codes) + ch);
    const float S = block_scale(scale_codes, c2, ch >> 1, fmt);
    const uint32_t words[4] = {cv.x, cv.y, cv.z, cv.w};
    if constexpr (sizeof(TOut) == 2) {
      uint32_t o[16];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t byte = (words[q] >> (8 * j)) & 0xffu;
          o[q * 4 + j] = pack_bf16x2(__fmul_rn(s_lv[byte & 0xf], S), __fmul_rn(s_lv[byte >> 4], S));
        }
      uint4 *dst = reinterpret_cast<uint4 *>(out + ch * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    } else {
      float o[32];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float p = __fmul_rn(s_lv[(words[q] >> (4 * j)) & 0xfu], S);
          o[q * 8 + j] = __uint_as_float(pack_bf16x2(p, 0.0f) << 16);
        }
      float4 *dst = reinterpret_cast<float4 *>(out + ch * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
  }
}

// bf16 output, coalesced without staging: a warp step is 4 segments of 256
// weights (128 bytes of codes, four 64-blocks).  Lane l decodes the 8 weights of
// code word l of each segment and stores them as one 16-byte write, so each of
// the warp's loads and stores covers 128 or 512 contiguous bytes.  The next
// step's codes and scales are loaded before this step's stores.
constexpr int kDequantWarps = kDequantThreads / 32;
__global__ void __launch_bounds__(kDequantThreads)
nf4_dequantize_bf16_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale_codes,
                           const float *__restrict__ c2, int64_t nweights, __nv_bfloat16 *__restrict__ out,
                           int fmt) {
  __shared__ float s_lv[16];
  if (threadIdx.x < 16) s_lv[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nwords = nweights / 8;       // 32-bit code words (8 weights each)
  const int64_t nsteps = (nweights + 1023) / 1024;
  const int64_t wstride = (int64_t)gridDim.x * kDequantWarps;
  int64_t ws = (int64_t)blockIdx.x * kDequantWarps + warp;
  uint32_t cw[4], sq[4];
  float cz[4];
  auto fetch = [&](int64_t step) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t w = (step * 4 + k) * 32 + lane;  // code word
      const bool in = step < nsteps && w < nwords;
      cw[k] = in ? __ldcs(reinterpret_cast<const uint32_t *>(codes) + w) : 0u;
      sq[k] = in ? __ldg(scale_codes + (w >> 3)) : 0u;
      cz[k] = in ? __ldg(c2 + (w >> 11)) : 0.0f;
    }
  };
  fetch(ws);
  for (; ws < nsteps; ws += wstride) {
    uint32_t wv[4];
    float S[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      wv[k] = cw[k];
      S[k] = __fmul_rn(scale_code_value(sq[k], fmt), cz[k]);
    }
    const int64_t w0 = ws * 128 + lane;  // this lane's first code word of the step
    fetch(ws + wstride);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t w = w0 + 32 * k;
      if (w < nwords) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t byte = (wv[k] >> (8 * j)) & 0xffu;
          o[j] = pack_bf16x2(__fmul_rn(s_lv[byte & 0xf], S[k]), __fmul_rn(s_lv[byte >> 4], S[k]));
        }
        __stcs(reinterpret_cast<uint4 *>(out + w * 8), make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}


// The same with 32-byte stores, for a 32-byte aligned output: each lane decodes
// two consecutive code words (16 weights of one block, one block scale) and
// writes them with one 256-bit store, so a warp instruction writes 1 KB.
__global__ void __launch_bounds__(kDequantThreads)
nf4_dequantize_bf16_v8_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale_codes,
                              const float *__restrict__ c2, int64_t nweights, __nv_bfloat16 *__restrict__ out,
                              int fmt) {
  __shared__ float s_lv[16];
  if (threadIdx.x < 16) s_lv[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nwords = nweights / 8;  // a multiple of 8 (whole blocks)
  const int64_t nsteps = (nweights + 1023) / 1024;
  const int64_t wstride = (int64_t)gridDim.x * kDequantWarps;
  int64_t ws = (int64_t)blockIdx.x * kDequantWarps + warp;
  uint2 cw[2];
  uint32_t sq[2];
  float cz[2];
  auto fetch = [&](int64_t step) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t w = step * 128 + k * 64 + 2 * lane;  // the lane's first code word of the pair
      const bool in = step < nsteps && w < nwords;
      cw[k] = in ? __ldcs(reinterpret_cast<const uint2 *>(codes) + w / 2) : make_uint2(0, 0);
      sq[k] = in ? __ldg(scale_codes + (w >> 3)) : 0u;
      cz[k] = in ? __ldg(c2 + (w >> 11)) : 0.0f;
    }
  };
  fetch(ws);
  for (; ws < nsteps; ws += wstride) {
    uint2 wv[2];
    float S[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      wv[k] = cw[k];
      S[k] = __fmul_rn(scale_code_value(sq[k], fmt), cz[k]);
    }
    const int64_t w0 = ws * 128 + 2 * lane;
    fetch(ws + wstride);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t w = w0 + 64 * k;
      if (w < nwords) {
        uint32_t o[8];
        const uint32_t ww[2] = {wv[k].x, wv[k].y};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t byte = (ww[h] >> (8 * j)) & 0xffu;
            o[4 * h + j] = pack_bf16x2(__fmul_rn(s_lv[byte & 0xf], S[k]), __fmul_rn(s_lv[byte >> 4], S[k]));
          }
        asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(out + w * 8), "r"(o[0]),
                     "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                     : "memory");
      }
    }
  }
}

}  // namespace qlora
