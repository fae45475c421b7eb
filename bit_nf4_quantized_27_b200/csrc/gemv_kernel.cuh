// Small-M (decode-shaped) forward of the NF4 linear layer with LoRA, M <= 16:
//   Y [M, N] = X W'^T + (s T) B^T,   T = X A^T computed by lora_down_small_kernel.
//
// HBM-bound: the packed codes (0.5 B/weight) dominate the traffic.  Two kernels
// share the decode below: nf4_gemv_bulk_kernel (the one used whenever
// N % 16 == 0 and K % 256 == 0, with K <= 4096 or a multiple of 4096) stages
// each 16-row group's codes and scales in shared memory by TMA; the fallback
// nf4_gemv_lora_kernel, for other shapes, loads them from HBM into registers with
// 8-byte vector loads.  Each byte (two codes) indexes a 256-entry table of fp16
// level pairs (L[lo], L[hi]) kept in shared memory with one copy per lane (each
// lane reads its own bank, so lookups never conflict); the pair is directly one
// register of an m16n8k16 tensor-core A fragment (rows = 16 weight rows).  The
// per-block scale S' = E4M3(q) * c2 multiplies the fp32 partial of each 64-weight
// block after its four MMAs.  X enters the MMA as fp16 after an exact per-token
// power-of-two scaling (every bf16 value inside the scaled range is an fp16
// value), undone on the partial sums.  The result equals X (L S')^T with L
// rounded to fp16 (relative 2^-12); it differs from X W'^T only by the bf16
// rounding of the dequantised weights W' = bf16(L S').
//
// Work split: 16 warps per CTA; warp w owns the w-th 256-wide slice of each
// 4096-wide K chunk and keeps that slice of X as MMA B fragments in registers.  The
// mapping of fragment registers to k inside a 64-block is permuted (thread quad q
// owns k in [16q, 16q+16) of every block) identically for W and X, which leaves
// the dot products unchanged and lets each thread load 8 contiguous code bytes per
// row and block.  Each CTA owns a set of 16-row groups; per-warp partials land in
// shared memory and are summed in a fixed order (deterministic).
#pragma once

#include <mutex>

#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

constexpr int kGemvMaxM = 16;
constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvMaxRG = 10;  // row groups of 16 per CTA

// Per-token adapters of a decode batch that serves several adapters on one base:
// token t uses A[t] [r, K], B[t] [N, r] and scale s[t].
struct MultiLora {
  const __nv_bfloat16 *A[kGemvMaxM];
  const __nv_bfloat16 *B[kGemvMaxM];
  float s[kGemvMaxM];
};

constexpr int kBulkMaxRG = 5;
constexpr int kBulkMaxStages = 6;
// Shared-memory placement of the staged kernel's buffers (absolute shared addresses).
struct BulkLayout {
  uint32_t lut, red[kBulkMaxRG], stage[kBulkMaxStages], bar, end;
};

struct GemvArgs {
  const uint8_t *codes;
  const uint8_t *scale_codes;
  const float *c2;
  int scale_format;         // qlora_scale_format of scale_codes
  int64_t N, K;
  int M;
  const __nv_bfloat16 *X;   // [M, K]
  const __nv_bfloat16 *sT;  // [M, r]  s * X A^T
  const __nv_bfloat16 *B;   // [N, r]
  int r;
  void *Y;
  int y_f32;
  float *partial;           // unused scratch slot (reserved)
  uint32_t *status;
  int rg_per_cta;
  int stages;               // bulk kernel: depth of the shared-memory ring
  int multi;                // 1: token t adds s[t] (x_t A_t^T) B_t^T with ml's adapters;
                            // 2: per-token adapters, base product only (the LoRA term follows
                            //    in lora_up_multi_kernel)
  BulkLayout lay;           // bulk kernel: placement computed on the host for a window at lay_base
  uint32_t lay_base;
  MultiLora ml;
};

inline size_t gemv_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Read-only shared-memory load and an MMA without `volatile`, so the compiler
// may reorder them for latency (both have no side effects beyond their outputs).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void mma_16816_f16_nv(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^e as a float (|e| <= 126).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Two bf16 (packed) times 2^-e, converted to packed fp16.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t v, float inv) {
  const __half2 h = __floats2half2_rn(bf16lo_to_f32(v) * inv, bf16hi_to_f32(v) * inv);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// Waits for the preceding kernel (programmatic dependent launch) and returns 0.
// Reads of what that kernel writes (s T) take their address from the result, so
// the compiler cannot schedule them before the wait (a read-only .nc load
// declares the data constant for the whole kernel, which lets it move).  They
// are .ca loads: the data no longer changes once the wait returns, and caching
// it in L1 keeps every warp of every CTA from going to the same L2 lines.
__device__ __forceinline__ uint32_t griddep_wait_token() {
  uint32_t z;
  asm volatile("griddepcontrol.wait;\n\tmov.u32 %0, 0;" : "=r"(z) : : "memory");
  return z;
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Fallback for shapes the staged kernel does not take: codes and scales are
// loaded straight into registers.
// smem: table [256][32] u32 | red [rg][16 warps][16 rows][16 tokens] f32
template <int NG>
__global__ void __launch_bounds__(kGemvThreads, 1) nf4_gemv_lora_kernel(const GemvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem_raw);
  float *red = reinterpret_cast<float *>(smem_raw + 256 * 32 * 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;

  // Pair table: entry v = (fp16 L[v & 15]) | (fp16 L[v >> 4]) << 16, one copy per lane.
  for (int i = tid; i < 256 * 32; i += kGemvThreads) {
    const int v = i >> 5;
    const __half2 h = __floats2half2_rn(__uint_as_float(kNf4LevelBits[v & 15]), __uint_as_float(kNf4LevelBits[v >> 4]));
    lut[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  const int num_rg = static_cast<int>((a.N + 15) / 16);
  const int rg0 = blockIdx.x * a.rg_per_cta;
  const int my_rg = max(0, min(a.rg_per_cta, num_rg - rg0));
  for (int i = tid; i < my_rg * kGemvWarps * 256; i += kGemvThreads) red[i] = 0.0f;
  __syncthreads();

  const int64_t nbk = a.K / 64;            // blocks per row
  const int64_t row_bytes = a.K / 2;
  const uint32_t lut_lane = static_cast<uint32_t>(__cvta_generic_to_shared(lut)) + lane * 4;
  const int nchunks = static_cast<int>((nbk + 63) / 64);

  for (int ch = 0; ch < nchunks; ++ch) {
    const int64_t kb0 = (int64_t)ch * 64 + warp * 4;  // first block of this warp's quad
    if (kb0 >= nbk) continue;
    const int nblk = static_cast<int>(nbk - kb0 < 4 ? nbk - kb0 : 4);
    // X fragments: token (g + 8*ng), k = kb*64 + 16q + 4s + {0..3}, as fp16 after
    // scaling token t's slice by 2^-e_t with max |x| * 2^-e_t in [2^14, 2^15).
    uint32_t xf[4][4][NG][2];
    float unscale[NG][2];  // 2^e of tokens 2q, 2q+1 (+8 ng): the C fragment columns
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const int t = g + 8 * ng;
      uint4 raw[4][2];
      uint32_t mx = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (j < nblk && t < a.M) {
          const uint4 *src = reinterpret_cast<const uint4 *>(a.X + (int64_t)t * a.K + (kb0 + j) * 64 + 16 * q);
          v0 = __ldg(src);
          v1 = __ldg(src + 1);
        }
        raw[j][0] = v0;
        raw[j][1] = v1;
        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v0.x & 0x7fff7fffu, v0.y & 0x7fff7fffu),
                                   __vmaxu2(v0.z & 0x7fff7fffu, v0.w & 0x7fff7fffu)));
        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v1.x & 0x7fff7fffu, v1.y & 0x7fff7fffu),
                                   __vmaxu2(v1.z & 0x7fff7fffu, v1.w & 0x7fff7fffu)));
      }
      uint32_t m16 = max(mx & 0xffffu, mx >> 16);
      m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
      m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 2));
      // bf16 bits -> exponent E with max in [2^(E-1), 2^E); e = E - 15, clamped
      const int E = m16 ? static_cast<int>((m16 >> 7) & 0xff) - 126 : 15;
      const int e = max(-100, min(100, E - 15));
      const float inv = pow2f(-e);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xf[j][0][ng][0] = bf16x2_to_f16x2_scaled(raw[j][0].x, inv);
        xf[j][0][ng][1] = bf16x2_to_f16x2_scaled(raw[j][0].y, inv);
        xf[j][1][ng][0] = bf16x2_to_f16x2_scaled(raw[j][0].z, inv);
        xf[j][1][ng][1] = bf16x2_to_f16x2_scaled(raw[j][0].w, inv);
        xf[j][2][ng][0] = bf16x2_to_f16x2_scaled(raw[j][1].x, inv);
        xf[j][2][ng][1] = bf16x2_to_f16x2_scaled(raw[j][1].y, inv);
        xf[j][3][ng][0] = bf16x2_to_f16x2_scaled(raw[j][1].z, inv);
        xf[j][3][ng][1] = bf16x2_to_f16x2_scaled(raw[j][1].w, inv);
      }
      // exponent of token (2q + i + 8 ng) lives in lane (2q + i) * 4
      unscale[ng][0] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q) * 4));
      unscale[ng][1] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q + 1) * 4));
    }

    // Software pipeline over this CTA's row groups: codes and scale bytes of the
    // next PD groups are in flight while the current one is decoded.
    struct Stage {
      uint2 c[4][2];   // [block][row half] 8 code bytes
      uint32_t q[2];   // 4 E4M3 scale bytes per row half (blocks kb0..kb0+3)
      float c2[2][2];  // c2 of the quad's first group and, if it crosses one, the next
      uint32_t split[2];  // blocks j >= split use c2[h][1]
    };
    const bool quad_ok = (nbk & 3) == 0 && nblk == 4;  // 4-byte scale loads are aligned
    auto load_stage = [&](int i, Stage &st) {
      const int64_t n0 = (int64_t)(rg0 + i) * 16;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = n0 + g + 8 * h;
        const bool rv = row < a.N;
        const uint8_t *cp = a.codes + row * row_bytes + kb0 * 32 + 8 * q;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st.c[j][h] = (rv && j < nblk) ? __ldg(reinterpret_cast<const uint2 *>(cp + 32 * j))
                                        : make_uint2(0x77777777u, 0x77777777u);
        const int64_t b0 = row * nbk + kb0;
        if (rv && quad_ok) {
          st.q[h] = __ldg(reinterpret_cast<const uint32_t *>(a.scale_codes + b0));
        } else {
          uint32_t w = 0;
          for (int j = 0; j < 4; ++j)
            if (rv && j < nblk) w |= static_cast<uint32_t>(__ldg(a.scale_codes + b0 + j)) << (8 * j);
          st.q[h] = w;
        }
        // a quad crosses at most one boundary between groups of 256 blocks
        const uint32_t left = 256u - static_cast<uint32_t>(b0 & 255);
        st.split[h] = left < 4u ? left : 4u;
        st.c2[h][0] = rv ? __ldg(a.c2 + (b0 >> 8)) : 0.0f;
        st.c2[h][1] = (rv && left < 4u && left < static_cast<uint32_t>(nblk)) ? __ldg(a.c2 + (b0 >> 8) + 1) : st.c2[h][0];
      }
    };
    // Two stages filled alternately: a stage is refilled only after it has been
    // consumed, so no register holding an in-flight load is ever copied.
    auto process = [&](int i, const Stage &cur) {
      // block scales of rows g (h=0) and g+8 (h=1)
      float S[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 f01 = scale_code_value2(cur.q[h], a.scale_format);
        const float2 f23 = scale_code_value2(cur.q[h] >> 16, a.scale_format);
        S[h][0] = __fmul_rn(f01.x, cur.c2[h][0]);
        S[h][1] = __fmul_rn(f01.y, cur.split[h] > 1 ? cur.c2[h][0] : cur.c2[h][1]);
        S[h][2] = __fmul_rn(f23.x, cur.split[h] > 2 ? cur.c2[h][0] : cur.c2[h][1]);
        S[h][3] = __fmul_rn(f23.y, cur.split[h] > 3 ? cur.c2[h][0] : cur.c2[h][1]);
      }
      float part[NG][4];
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) part[ng][0] = part[ng][1] = part[ng][2] = part[ng][3] = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float acc[NG][4];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // bytes 2s, 2s+1 of the 8 code bytes of rows g (h=0) and g+8 (h=1)
          const uint32_t w0 = (s < 2) ? cur.c[j][0].x : cur.c[j][0].y;
          const uint32_t w1 = (s < 2) ? cur.c[j][1].x : cur.c[j][1].y;
          const uint32_t p0 = (2 * s) & 3, p1 = (2 * s + 1) & 3;
          const uint32_t b00 = __byte_perm(w0, 0u, 0x4440u | p0), b01 = __byte_perm(w0, 0u, 0x4440u | p1);
          const uint32_t b10 = __byte_perm(w1, 0u, 0x4440u | p0), b11 = __byte_perm(w1, 0u, 0x4440u | p1);
          uint32_t a0, a1, a2, a3;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(lut_lane + (b00 << 7)));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(lut_lane + (b10 << 7)));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(lut_lane + (b01 << 7)));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a3) : "r"(lut_lane + (b11 << 7)));
#pragma unroll
          for (int ng = 0; ng < NG; ++ng) mma_16816_f16(acc[ng], a0, a1, a2, a3, xf[j][s][ng][0], xf[j][s][ng][1]);
        }
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
          part[ng][0] = fmaf(S[0][j], acc[ng][0], part[ng][0]);
          part[ng][1] = fmaf(S[0][j], acc[ng][1], part[ng][1]);
          part[ng][2] = fmaf(S[1][j], acc[ng][2], part[ng][2]);
          part[ng][3] = fmaf(S[1][j], acc[ng][3], part[ng][3]);
        }
      }
      // red[i][warp][row][token] += partial * 2^e (this warp is the only writer)
      float *rb = red + ((size_t)i * kGemvWarps + warp) * 256;
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = 2 * q + 8 * ng;
        rb[g * 16 + t] += part[ng][0] * unscale[ng][0];
        rb[g * 16 + t + 1] += part[ng][1] * unscale[ng][1];
        rb[(g + 8) * 16 + t] += part[ng][2] * unscale[ng][0];
        rb[(g + 8) * 16 + t + 1] += part[ng][3] * unscale[ng][1];
      }
    };
    Stage sa, sb;
    if (my_rg > 0) load_stage(0, sa);
    for (int i = 0; i < my_rg; i += 2) {
      if (i + 1 < my_rg) load_stage(i + 1, sb);
      process(i, sa);
      if (i + 1 >= my_rg) break;
      if (i + 2 < my_rg) load_stage(i + 2, sa);
      process(i + 1, sb);
    }
  }

  // LoRA up-projection on tensor cores: rows = 16 weight rows (A = B_lora rows),
  // cols = tokens (B = (s T)^T), K = r.  Needs s T from the preceding kernel.
  const __nv_bfloat16 *const sT = a.sT + griddep_wait_token();
  for (int i = warp; i < my_rg; i += kGemvWarps) {
    const int64_t n0 = (int64_t)(rg0 + i) * 16;
    float acc[NG][4];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
    for (int j0 = 0; j0 < a.r; j0 += 16) {
      // A fragment: rows g / g+8, k = j0 + 2q + {0,1} and j0 + 8 + 2q + {0,1}
      uint32_t af[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = n0 + g + 8 * h;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(a.B + row * a.r + j0 + 2 * q);
        af[h] = (row < a.N && j0 + 2 * q < a.r) ? __ldg(src) : 0u;
        af[2 + h] = (row < a.N && j0 + 8 + 2 * q < a.r) ? __ldg(src + 4) : 0u;
      }
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = g + 8 * ng;
        uint32_t b0 = 0, b1 = 0;
        if (t < a.M) {
          const unsigned *src = reinterpret_cast<const unsigned *>(sT + (int64_t)t * a.r + j0 + 2 * q);
          if (j0 + 2 * q < a.r) b0 = __ldca(src);
          if (j0 + 8 + 2 * q < a.r) b1 = __ldca(src + 4);
        }
        mma_16816(acc[ng], af[0], af[1], af[2], af[3], b0, b1);
      }
    }
    float *rb = red + ((size_t)i * kGemvWarps + warp) * 256;
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const int t = 2 * q + 8 * ng;
      rb[g * 16 + t] += acc[ng][0];
      rb[g * 16 + t + 1] += acc[ng][1];
      rb[(g + 8) * 16 + t] += acc[ng][2];
      rb[(g + 8) * 16 + t + 1] += acc[ng][3];
    }
  }
  __syncthreads();

  // Deterministic reduction over the 16 warps and store.
  for (int idx = tid; idx < my_rg * 256; idx += kGemvThreads) {
    const int i = idx >> 8, e = idx & 255, row = e >> 4, t = e & 15;
    const int64_t n = (int64_t)(rg0 + i) * 16 + row;
    if (t >= a.M || n >= a.N) continue;
    const float *rb = red + (size_t)i * kGemvWarps * 256 + e;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) sum += rb[w * 256];
    if (a.y_f32) reinterpret_cast<float *>(a.Y)[(int64_t)t * a.N + n] = sum;
    else reinterpret_cast<__nv_bfloat16 *>(a.Y)[(int64_t)t * a.N + n] = __float2bfloat16_rn(sum);
  }
}

// ---------------------------------------------------------------------------
// Bulk-staged variant: each 16-row group's codes (16 x CH/2 bytes, one 3-D TMA
// copy) and block scales (16 x CH/64 bytes, one bulk copy) arrive in shared
// memory in a ring of up to kBulkMaxStages stages, so DRAM sees long contiguous
// reads and up to about 130 KB stays in flight per SM without holding
// registers.  Both copies carry an L2 evict-first policy: a decode step reads
// each weight once.  Requirements: N % 16 == 0, K % 256 == 0 and (K <= 4096 or
// K % 4096 == 0); CH = min(K, 4096).
// ---------------------------------------------------------------------------

__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
      "l"(src), "r"(bytes), "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "l"(policy)
      : "memory");
}

inline bool gemv_bulk_ok(int64_t N, int64_t K) {
  return N % 16 == 0 && K % 256 == 0 && (K <= 4096 || K % 4096 == 0);
}

// Shared memory of the bulk kernel.  The pair table sits at a 64 KB-aligned
// shared address with a 256-byte row per byte value (a lane's entry at
// row * 256 + lane * 4), so one byte permute builds the whole lookup address:
// [lane * 4 | code byte | table base bits 16..31].  The stage ring, the
// row-group partial sums and the barriers are placed before the table where
// they fit and after it otherwise.
constexpr uint32_t kBulkLutBytes = 256 * 256;
constexpr uint32_t kBulkSmemLimit = 232448;  // opt-in dynamic shared memory per CTA

// A stage holds one 16-row group's codes for a chunk of CH = min(K, 4096)
// columns, brought in by one 3-D TMA copy (128 bytes x 16 rows x CH/256
// column chunks) with the 128-byte swizzle: shared layout [chunk][row][128 B]
// with each 16-byte unit's index XORed with (row & 7), so the eight rows one
// warp reads in an instruction land in different banks.  The stage's block
// scales (16 rows x CH/64 bytes, row-major) follow the codes.
__host__ __device__ inline uint32_t gemv_bulk_stage_bytes(int64_t K) {
  const int64_t CH = K < 4096 ? K : 4096;
  return static_cast<uint32_t>((16 * CH / 2 + 16 * CH / 64 + 1023) & ~int64_t(1023));
}
// Partial sums of one row group: [16 warps][16 rows][TR tokens] floats, TR = M
// for M <= 8 (one n8 tile), else 16.
__host__ __device__ inline int gemv_bulk_red_tokens(int M) { return M <= 8 ? M : 16; }
__host__ __device__ inline uint32_t gemv_bulk_red_bytes(int M) {
  return static_cast<uint32_t>(kGemvWarps * 16 * gemv_bulk_red_tokens(M) * 4);
}

// Placement of the bulk kernel's buffers around the 64 KB-aligned table, for a
// dynamic window starting at shared address `base` (computed on the host and
// passed to the kernel, which checks that its window starts there).
__host__ __device__ inline BulkLayout gemv_bulk_layout(uint32_t base, uint32_t stage_bytes, int stages,
                                                       uint32_t red_bytes) {
  BulkLayout L;
  L.lut = (base + 0xffffu) & ~0xffffu;
  uint32_t lo_next = base, hi_next = L.lut + kBulkLutBytes;
  auto place = [&](uint32_t bytes, uint32_t align) -> uint32_t {
    const uint32_t lo = (lo_next + align - 1) & ~(align - 1);
    if (lo + bytes <= L.lut) {
      lo_next = lo + bytes;
      return lo;
    }
    const uint32_t hi = (hi_next + align - 1) & ~(align - 1);
    hi_next = hi + bytes;
    return hi;
  };
  for (int i = 0; i < kBulkMaxStages; ++i) L.stage[i] = i < stages ? place(stage_bytes, 1024) : 0u;
  for (int i = 0; i < kBulkMaxRG; ++i) L.red[i] = place(red_bytes, 16);
  L.bar = place(2 * kBulkMaxStages * 8, 16);
  L.end = hi_next > lo_next ? hi_next : lo_next;
  return L;
}

inline int gemv_bulk_smem_bytes(int64_t K, int stages, int M, uint32_t base) {
  const BulkLayout L = gemv_bulk_layout(base, gemv_bulk_stage_bytes(K), stages, gemv_bulk_red_bytes(M));
  return static_cast<int>(L.end - base);
}

// Largest stage count (at most `uses`, the stages one CTA consumes, but at least
// two) whose layout fits a dynamic window starting at `base`; 0 if two do not fit.
inline int gemv_bulk_stages(int64_t K, int M, uint32_t base, int uses) {
  const int top = uses < 2 ? 2 : (uses > kBulkMaxStages ? kBulkMaxStages : uses);
  for (int s = top; s >= 2; --s)
    if (gemv_bulk_smem_bytes(K, s, M, base) <= static_cast<int>(kBulkSmemLimit)) return s;
  return 0;
}

template <int NG>
__global__ void __launch_bounds__(kGemvThreads, 1)
    nf4_gemv_bulk_kernel(const __grid_constant__ CUtensorMap tm_codes, const GemvArgs a, int dyn_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int64_t CH = a.K < 4096 ? a.K : 4096;
  const int S = a.stages;
  const int TR = gemv_bulk_red_tokens(a.M);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  if (tid == 0) ptx::prefetch_tmap(&tm_codes);

  // ---- layout around the 64 KB-aligned table, placed by the host for the
  // window start it expects (recomputing it here costs a noticeable share of a
  // decode call's few microseconds)
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const BulkLayout &Lay = a.lay;
  if (base != a.lay_base || S < 2 || S > kBulkMaxStages || Lay.end > base + static_cast<uint32_t>(dyn_bytes)) {
    if (tid == 0) raise_status(a.status, QLORA_ERR_CUDA);  // the host sized the window for another start
    return;
  }
  const uint32_t lut_addr = Lay.lut;
  auto at = [&](uint32_t addr) { return smem_raw + (addr - base); };
  // run-time indices pick addresses by selects, keeping the layout in registers
  auto stage_at = [&](int slot) {
    uint32_t v = Lay.stage[0];
#pragma unroll
    for (int k = 1; k < kBulkMaxStages; ++k) v = slot == k ? Lay.stage[k] : v;
    return at(v);
  };
  auto red_at = [&](int i) {
    uint32_t v = Lay.red[0];
#pragma unroll
    for (int k = 1; k < kBulkMaxRG; ++k) v = i == k ? Lay.red[k] : v;
    return reinterpret_cast<float *>(at(v));
  };
  uint64_t *full = reinterpret_cast<uint64_t *>(at(Lay.bar));
  uint64_t *empty = full + kBulkMaxStages;

  const int num_rg = static_cast<int>(a.N / 16);
  const int rg0 = blockIdx.x * a.rg_per_cta;
  const int my_rg = max(0, min(a.rg_per_cta, num_rg - rg0));
  const int64_t nbk = a.K / 64;
  const int nch = static_cast<int>(a.K / CH);
  const int total = my_rg * nch;
  const int nw = static_cast<int>(CH / 256);  // warps with columns in a chunk
  const bool active = warp < nw;

  // producer (thread 0): stage u = (chunk u / my_rg, row group u % my_rg); the
  // codes and block scales are read once per call, so they enter L2 as evict-first
  const uint64_t policy = ptx::l2_evict_first_policy();
  auto issue = [&](int u) {
    const int ch = u / my_rg, i = u % my_rg;
    const int slot = u % S;
    uint8_t *st = stage_at(slot);
    const int64_t n0 = (int64_t)(rg0 + i) * 16;
    ptx::mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(16 * CH / 2 + 16 * CH / 64));
    ptx::tma_load_3d_hint(st, &tm_codes, &full[slot], 0, static_cast<int32_t>(n0),
                          ch * static_cast<int32_t>(CH / 256), policy);
    if (CH == a.K) {
      bulk_g2s_hint(st + 16 * CH / 2, a.scale_codes + n0 * nbk, static_cast<uint32_t>(16 * nbk), &full[slot], policy);
    } else {
      for (int rw = 0; rw < 16; ++rw)
        bulk_g2s_hint(st + 16 * CH / 2 + rw * (CH / 64), a.scale_codes + (n0 + rw) * nbk + ch * (CH / 64),
                      static_cast<uint32_t>(CH / 64), &full[slot], policy);
    }
  };
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kGemvThreads);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int u = 0; u < S && u < total; ++u) issue(u);
  // per-token adapters: each token's B rows of this CTA's row groups (contiguous,
  // my_rg * 16 rows of r ranks) start moving into L2 now, behind the weight stream,
  // so that the LoRA step after the main loop reads them from L2
  if (a.multi == 1 && warp == 1 && lane < a.M && my_rg > 0)
    ptx::bulk_prefetch_l2(a.ml.B[lane] + (int64_t)rg0 * 16 * a.r, static_cast<uint32_t>(my_rg * 16 * a.r * 2));

  // this warp's slice of X for a chunk (raw bf16)
  uint4 xraw[NG][4][2];
  auto load_x = [&](int ch) {
    const int64_t kb0 = (int64_t)ch * 64 + warp * 4;
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const int t = g + 8 * ng;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (active && t < a.M) {
          const uint4 *src = reinterpret_cast<const uint4 *>(a.X + (int64_t)t * a.K + (kb0 + j) * 64 + 16 * q);
          v0 = __ldg(src);
          v1 = __ldg(src + 1);
        }
        xraw[ng][j][0] = v0;
        xraw[ng][j][1] = v1;
      }
    }
  };
  // pair table: row v, lane l holds fp16 (L[v & 15], L[v >> 4]) at v*256 + l*4;
  // four lanes' identical entries per 16-byte store
  for (int i = tid; i < 256 * 8; i += kGemvThreads) {
    const int v = i >> 3;
    const __half2 h = __floats2half2_rn(__uint_as_float(kNf4LevelBits[v & 15]), __uint_as_float(kNf4LevelBits[v >> 4]));
    const uint32_t e = *reinterpret_cast<const uint32_t *>(&h);
    *reinterpret_cast<uint4 *>(at(lut_addr + v * 256 + (i & 7) * 16)) = make_uint4(e, e, e, e);
  }
  __syncthreads();
  // [lane * 4, -, table base bits 16..23, 24..31]: the byte permute inserts the code byte
  const uint32_t laneword = (lut_addr & 0xffff0000u) | static_cast<uint32_t>(lane * 4);
  // this thread's 8 code bytes of block 4*warp + j, row g (+8 for h = 1): chunk
  // `warp`, line offset 32j + 8q, 16-byte unit (2j + q/2) XOR g
  const uint32_t code_off = warp * 2048 + g * 128 + 8 * (q & 1);
  uint32_t code_xo[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) code_xo[j] = static_cast<uint32_t>(((2 * j + (q >> 1)) ^ g) << 4);
  bool ok = true;

  for (int ch = 0; ch < nch && ok; ++ch) {
    const int64_t kb0 = (int64_t)ch * 64 + warp * 4;  // first block of this warp's quad (global)
    load_x(ch);
    uint32_t xf[4][4][NG][2];
    float unscale[NG][2];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const uint4(&raw)[4][2] = xraw[ng];
      uint32_t mx = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v0 = raw[j][0], v1 = raw[j][1];
        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v0.x & 0x7fff7fffu, v0.y & 0x7fff7fffu),
                                   __vmaxu2(v0.z & 0x7fff7fffu, v0.w & 0x7fff7fffu)));
        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v1.x & 0x7fff7fffu, v1.y & 0x7fff7fffu),
                                   __vmaxu2(v1.z & 0x7fff7fffu, v1.w & 0x7fff7fffu)));
      }
      uint32_t m16 = max(mx & 0xffffu, mx >> 16);
      m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
      m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 2));
      const int E = m16 ? static_cast<int>((m16 >> 7) & 0xff) - 126 : 15;
      const int e = max(-100, min(100, E - 15));
      const float inv = pow2f(-e);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xf[j][0][ng][0] = bf16x2_to_f16x2_scaled(raw[j][0].x, inv);
        xf[j][0][ng][1] = bf16x2_to_f16x2_scaled(raw[j][0].y, inv);
        xf[j][1][ng][0] = bf16x2_to_f16x2_scaled(raw[j][0].z, inv);
        xf[j][1][ng][1] = bf16x2_to_f16x2_scaled(raw[j][0].w, inv);
        xf[j][2][ng][0] = bf16x2_to_f16x2_scaled(raw[j][1].x, inv);
        xf[j][2][ng][1] = bf16x2_to_f16x2_scaled(raw[j][1].y, inv);
        xf[j][3][ng][0] = bf16x2_to_f16x2_scaled(raw[j][1].z, inv);
        xf[j][3][ng][1] = bf16x2_to_f16x2_scaled(raw[j][1].w, inv);
      }
      unscale[ng][0] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q) * 4));
      unscale[ng][1] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q + 1) * 4));
    }

    auto c2_of = [&](int i, float (&c)[2]) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = (int64_t)(rg0 + i) * 16 + g + 8 * h;
        c[h] = active ? __ldg(a.c2 + ((row * nbk + kb0) >> 8)) : 0.0f;
      }
    };
    auto release = [&](int u, int slot) -> bool {
      ptx::mbar_arrive(&empty[slot]);
      if (tid == 0 && u + S < total) {
        if (!ptx::mbar_wait(&empty[slot], (u / S) & 1, nullptr)) return false;
        issue(u + S);
      }
      return true;
    };
    auto process = [&](int i, const float (&c2v)[2]) -> bool {
      const int u = ch * my_rg + i;
      const int slot = u % S;
      if (!ptx::mbar_wait(&full[slot], (u / S) & 1, nullptr)) return false;
      if (!active) return release(u, slot);
      const uint8_t *st = stage_at(slot);
      const int kl = warp * 4;  // quad's first block within the chunk
      uint2 cw[4][2];
      uint32_t qw[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rw = g + 8 * h;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          cw[j][h] = *reinterpret_cast<const uint2 *>(st + code_off + h * 1024 + code_xo[j]);
        qw[h] = *reinterpret_cast<const uint32_t *>(st + 16 * CH / 2 + rw * (CH / 64) + kl);
      }
      if (!release(u, slot)) return false;
      float S4[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 f01 = scale_code_value2(qw[h], a.scale_format);
        const float2 f23 = scale_code_value2(qw[h] >> 16, a.scale_format);
        S4[h][0] = __fmul_rn(f01.x, c2v[h]);
        S4[h][1] = __fmul_rn(f01.y, c2v[h]);
        S4[h][2] = __fmul_rn(f23.x, c2v[h]);
        S4[h][3] = __fmul_rn(f23.y, c2v[h]);
      }
      float part[NG][4];
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) part[ng][0] = part[ng][1] = part[ng][2] = part[ng][3] = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float acc[NG][4];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
        // all 16 table lookups of the block first, then its 4 MMAs (the table
        // is read-only here, so these loads may be scheduled freely)
        uint32_t af[4][4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t w0 = (s < 2) ? cw[j][0].x : cw[j][0].y;
          const uint32_t w1 = (s < 2) ? cw[j][1].x : cw[j][1].y;
          const uint32_t p0 = (2 * s) & 3, p1 = (2 * s + 1) & 3;
          af[s][0] = lds_u32(__byte_perm(w0, laneword, 0x7604u | (p0 << 4)));
          af[s][1] = lds_u32(__byte_perm(w1, laneword, 0x7604u | (p0 << 4)));
          af[s][2] = lds_u32(__byte_perm(w0, laneword, 0x7604u | (p1 << 4)));
          af[s][3] = lds_u32(__byte_perm(w1, laneword, 0x7604u | (p1 << 4)));
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
          for (int ng = 0; ng < NG; ++ng)
            mma_16816_f16_nv(acc[ng], af[s][0], af[s][1], af[s][2], af[s][3], xf[j][s][ng][0], xf[j][s][ng][1]);
        }
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
          part[ng][0] = fmaf(S4[0][j], acc[ng][0], part[ng][0]);
          part[ng][1] = fmaf(S4[0][j], acc[ng][1], part[ng][1]);
          part[ng][2] = fmaf(S4[1][j], acc[ng][2], part[ng][2]);
          part[ng][3] = fmaf(S4[1][j], acc[ng][3], part[ng][3]);
        }
      }
      // this warp's slot of row group i: written by the first chunk, accumulated by later ones
      float *rb = red_at(i) + warp * 16 * TR;
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = 2 * q + 8 * ng;
        const float v00 = part[ng][0] * unscale[ng][0], v01 = part[ng][1] * unscale[ng][1];
        const float v10 = part[ng][2] * unscale[ng][0], v11 = part[ng][3] * unscale[ng][1];
        if (ch == 0) {
          if (t < TR) rb[g * TR + t] = v00, rb[(g + 8) * TR + t] = v10;
          if (t + 1 < TR) rb[g * TR + t + 1] = v01, rb[(g + 8) * TR + t + 1] = v11;
        } else {
          if (t < TR) rb[g * TR + t] += v00, rb[(g + 8) * TR + t] += v10;
          if (t + 1 < TR) rb[g * TR + t + 1] += v01, rb[(g + 8) * TR + t + 1] += v11;
        }
      }
      return true;
    };
    // one copy of the row-group body (the loop is not unrolled), so the
    // instruction footprint of the steady state stays small
    float cn[2] = {0.0f, 0.0f};
    if (my_rg > 0) c2_of(0, cn);
#pragma unroll 1
    for (int i = 0; i < my_rg && ok; ++i) {
      const float cc[2] = {cn[0], cn[1]};
      if (i + 1 < my_rg) c2_of(i + 1, cn);
      ok = process(i, cc);
    }
  }
  if (!ok && lane == 0) raise_status(a.status, QLORA_ERR_TIMEOUT);

  // LoRA up-projection, added to warp 0's slot of each row group once every
  // warp has written its own.  B rows are loaded before the barrier, s T after
  // waiting for the kernel that computes it.
  const int lora_rg = warp < my_rg ? warp : -1;
  uint32_t bfr[4][4];
  if (lora_rg >= 0 && !a.multi) {
    const int64_t n0 = (int64_t)(rg0 + lora_rg) * 16;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j0 = 16 * jj;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(a.B + (n0 + g + 8 * h) * a.r + j0 + 2 * q);
        bfr[jj][h] = (j0 + 2 * q < a.r) ? __ldg(src) : 0u;
        bfr[jj][2 + h] = (j0 + 8 + 2 * q < a.r) ? __ldg(src + 4) : 0u;
      }
    }
  }
  __syncthreads();
  const __nv_bfloat16 *const sT = a.sT + griddep_wait_token();
  if (a.multi == 1) {
    // one adapter per token.  s T (all tokens) is copied to shared memory (the
    // pair table's space, unused after the main loop).  Each token's B rows of
    // this CTA's row groups are one contiguous block of 16-byte pieces (P = r / 8
    // per row).
    uint4 *sts = reinterpret_cast<uint4 *>(at(lut_addr));
    const int P = a.r / 8;  // r % 8 == 0
    const int n16 = a.M * P;
    for (int i = tid; i < n16; i += kGemvThreads) sts[i] = __ldcg(reinterpret_cast<const uint4 *>(sT) + i);
    __syncthreads();
    if ((P & (P - 1)) == 0) {
      // P a power of two (r = 8, 16, 32, 64, 128, 256): every warp reads 32
      // consecutive pieces per load (coalesced), eight loads in flight per lane;
      // the P lanes of a row (an aligned group, never split across rows or
      // tokens) combine their partial dots by a butterfly in fixed order, and the
      // first adds the row's sum to its token's column.
      constexpr int U = 8;
      const int lgP = __ffs(P) - 1;
      const int per_t = (my_rg * 16) << lgP;  // pieces per token (at most 5 * 16 * 32)
      const int total = a.M * per_t;           // below 2^16
      // piece / per_t as a multiply-high: exact while piece * per_t < 2^32
      const uint32_t inv_t = 0xffffffffu / static_cast<uint32_t>(max(per_t, 1)) + 1u;
      for (int b0 = warp * 32 + lane; b0 - lane < total; b0 += kGemvThreads * U) {  // warp-uniform test
        uint4 bv[U];
        int tk[U], pr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int pp = b0 + u * kGemvThreads;
          const int pc = pp < total ? pp : total - 1;  // past the end: the last piece again, not summed
          const int t = static_cast<int>(__umulhi(static_cast<uint32_t>(pc), inv_t));
          tk[u] = t;
          pr[u] = pc - t * per_t;
          bv[u] = __ldg(reinterpret_cast<const uint4 *>(a.ml.B[t] + (int64_t)rg0 * 16 * a.r) + pr[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int ch = pr[u] & (P - 1);
          const uint4 sv = sts[tk[u] * P + ch];
          const uint32_t bw[4] = {bv[u].x, bv[u].y, bv[u].z, bv[u].w};
          const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
          float v = 0.0f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v = fmaf(bf16lo_to_f32(bw[e]), bf16lo_to_f32(sw[e]), v);
            v = fmaf(bf16hi_to_f32(bw[e]), bf16hi_to_f32(sw[e]), v);
          }
          for (int o = 1; o < P; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          const int rrow = pr[u] >> lgP;
          if (ch == 0 && b0 + u * kGemvThreads < total)
            red_at(rrow >> 4)[(rrow & 15) * TR + tk[u]] += v;  // warp 0's slot of the row group
        }
      }
    } else {
    const int row = lane & 15, nh = 2 * kGemvWarps;
    const int ntask = my_rg * a.M;
    for (int k0 = 2 * warp + (lane >> 4); k0 < ntask; k0 += 2 * nh) {
      int ti[2], tt[2];
      bool live[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int k = k0 + u * nh;
        live[u] = k < ntask;
        ti[u] = live[u] ? k / a.M : 0;  // a task past the end reads row group 0 of token 0, unused
        tt[u] = live[u] ? k - ti[u] * a.M : 0;
      }
      float acc[2] = {0.0f, 0.0f};
      for (int j0 = 0; j0 < a.r; j0 += 64) {
        // 64 ranks per round: eight 16-byte loads per task, all issued before the
        // products; loads past rank r re-read the round's last piece (in bounds)
        // and are not summed
        const int cl = min(8, (a.r - j0) / 8) - 1;
        uint4 bv[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int64_t n = (int64_t)(rg0 + ti[u]) * 16 + row;
          const uint4 *src = reinterpret_cast<const uint4 *>(a.ml.B[tt[u]] + n * a.r + j0);
#pragma unroll
          for (int c = 0; c < 8; ++c) bv[u][c] = __ldg(src + min(c, cl));
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint4 *st = sts + (tt[u] * a.r + j0) / 8;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (c > cl) break;
            const uint4 sv = st[c];
            const uint32_t bw[4] = {bv[u][c].x, bv[u][c].y, bv[u][c].z, bv[u][c].w};
            const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[u] = fmaf(bf16lo_to_f32(bw[e]), bf16lo_to_f32(sw[e]), acc[u]);
              acc[u] = fmaf(bf16hi_to_f32(bw[e]), bf16hi_to_f32(sw[e]), acc[u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (live[u]) red_at(ti[u])[row * TR + tt[u]] += acc[u];  // warp 0's slot of row group ti
    }
    }
  }
  if (lora_rg >= 0 && !a.multi) {
    const int64_t n0 = (int64_t)(rg0 + lora_rg) * 16;
    float acc[NG][4];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
    // the first 64 ranks: every s T fragment loaded at once, then the MMAs
    uint32_t bt[4][NG][2];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j0 = 16 * jj;
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = g + 8 * ng;
        const unsigned *src = reinterpret_cast<const unsigned *>(sT + (int64_t)t * a.r + j0 + 2 * q);
        bt[jj][ng][0] = (t < a.M && j0 + 2 * q < a.r) ? __ldca(src) : 0u;
        bt[jj][ng][1] = (t < a.M && j0 + 8 + 2 * q < a.r) ? __ldca(src + 4) : 0u;
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int ng = 0; ng < NG; ++ng)
        mma_16816(acc[ng], bfr[jj][0], bfr[jj][1], bfr[jj][2], bfr[jj][3], bt[jj][ng][0], bt[jj][ng][1]);
    for (int j0 = 64; j0 < a.r; j0 += 16) {
      uint32_t af[4];
      {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t *src = reinterpret_cast<const uint32_t *>(a.B + (n0 + g + 8 * h) * a.r + j0 + 2 * q);
          af[h] = (j0 + 2 * q < a.r) ? __ldg(src) : 0u;
          af[2 + h] = (j0 + 8 + 2 * q < a.r) ? __ldg(src + 4) : 0u;
        }
      }
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = g + 8 * ng;
        uint32_t b0 = 0, b1 = 0;
        if (t < a.M) {
          const unsigned *src = reinterpret_cast<const unsigned *>(sT + (int64_t)t * a.r + j0 + 2 * q);
          if (j0 + 2 * q < a.r) b0 = __ldca(src);
          if (j0 + 8 + 2 * q < a.r) b1 = __ldca(src + 4);
        }
        mma_16816(acc[ng], af[0], af[1], af[2], af[3], b0, b1);
      }
    }
    float *rb = red_at(lora_rg);  // warp 0's slot
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const int t = 2 * q + 8 * ng;
      if (t < TR) rb[g * TR + t] += acc[ng][0], rb[(g + 8) * TR + t] += acc[ng][2];
      if (t + 1 < TR) rb[g * TR + t + 1] += acc[ng][1], rb[(g + 8) * TR + t + 1] += acc[ng][3];
    }
  }
  __syncthreads();
  // deterministic sum over the warps that hold columns, in warp order
  const int per_rg = 16 * a.M;
  for (int idx = tid; idx < my_rg * per_rg; idx += kGemvThreads) {
    const int i = idx / per_rg, e = idx - i * per_rg, row = e / a.M, t = e - row * a.M;
    const int64_t n = (int64_t)(rg0 + i) * 16 + row;
    const float *rb = red_at(i) + row * TR + t;
    float sum = 0.0f;
    for (int w = 0; w < nw; ++w) sum += rb[w * 16 * TR];
    if (a.y_f32) reinterpret_cast<float *>(a.Y)[(int64_t)t * a.N + n] = sum;
    else reinterpret_cast<__nv_bfloat16 *>(a.Y)[(int64_t)t * a.N + n] = __float2bfloat16_rn(sum);
  }
}

// T = X A^T for M <= 16 tokens on tensor cores, in few CTAs so that it runs on
// SMs the decode GEMV leaves free.  CTA c computes rank rows [16c, 16c + 16):
// 8 warps split K in 64-column blocks (warp w takes blocks w, w + 8, ...), each
// runs m16n8k16 MMAs with A = 16 rows of the LoRA A matrix and B = X^T (tokens),
// both bf16.  Inside a block, k is permuted identically for A and X (thread quad
// q owns k in [16q, 16q + 16)), so each thread reads two 16-byte vectors per row
// and block, and a warp has kLoraDownBlocks blocks of loads in flight before its
// first MMA.  The partials are summed over the warps in a fixed order and
// multiplied by t_scale (1, or 1 / (1 - p) for a dropped-out X).  Writes s*T
// (bf16) and, if T_hi is given, (T_hi, T_lo).
constexpr int kLoraDownThreads = 256;
constexpr int kLoraDownBlocks = 4;
template <int NG>
__global__ void __launch_bounds__(kLoraDownThreads, 1) lora_down_small_kernel(
    const __nv_bfloat16 *__restrict__ X, const __nv_bfloat16 *__restrict__ A, int M, int64_t K, int r, float s,
    __nv_bfloat16 *__restrict__ sT, __nv_bfloat16 *__restrict__ T_hi, __nv_bfloat16 *__restrict__ T_lo,
    float t_scale) {
  griddep_launch_dependents();
  __shared__ float red[kLoraDownThreads / 32][16][kGemvMaxM];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int j0 = blockIdx.x * 16;
  const int64_t nb = K / 64;
  float acc[NG][4];
#pragma unroll
  for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
  const bool rv[2] = {j0 + g < r, j0 + g + 8 < r};
  for (int64_t kb0 = warp; kb0 < nb; kb0 += (kLoraDownThreads / 32) * kLoraDownBlocks) {
    uint4 av[kLoraDownBlocks][2][2], xv[kLoraDownBlocks][NG][2];
#pragma unroll
    for (int u = 0; u < kLoraDownBlocks; ++u) {
      const int64_t kb = kb0 + (kLoraDownThreads / 32) * u;
      const bool kin = kb < nb;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 *src = reinterpret_cast<const uint4 *>(A + (int64_t)(j0 + g + 8 * h) * K + kb * 64 + 16 * q);
        av[u][h][0] = (kin && rv[h]) ? __ldg(src) : make_uint4(0, 0, 0, 0);
        av[u][h][1] = (kin && rv[h]) ? __ldg(src + 1) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = g + 8 * ng;
        const uint4 *src = reinterpret_cast<const uint4 *>(X + (int64_t)t * K + kb * 64 + 16 * q);
        xv[u][ng][0] = (kin && t < M) ? __ldg(src) : make_uint4(0, 0, 0, 0);
        xv[u][ng][1] = (kin && t < M) ? __ldg(src + 1) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kLoraDownBlocks; ++u) {
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        // step st uses k = 16q + 4st + {0, 1} (fragment slots 2q, 2q+1) and + {2, 3} (slots 2q+8, 2q+9)
        const int hv = st >> 1;
        const bool zw = st & 1;
        const uint32_t a0 = zw ? av[u][0][hv].z : av[u][0][hv].x, a2 = zw ? av[u][0][hv].w : av[u][0][hv].y;
        const uint32_t a1 = zw ? av[u][1][hv].z : av[u][1][hv].x, a3 = zw ? av[u][1][hv].w : av[u][1][hv].y;
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) {
          const uint32_t b0 = zw ? xv[u][ng][hv].z : xv[u][ng][hv].x, b1 = zw ? xv[u][ng][hv].w : xv[u][ng][hv].y;
          mma_16816(acc[ng], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
  // C fragment: rows g / g+8 (rank), columns 2q, 2q+1 (+8 ng) (tokens)
#pragma unroll
  for (int ng = 0; ng < 2; ++ng) {
    const int t = 2 * q + 8 * ng;
    const bool have = ng < NG;
    red[warp][g][t] = have ? acc[ng < NG ? ng : 0][0] : 0.0f;
    red[warp][g][t + 1] = have ? acc[ng < NG ? ng : 0][1] : 0.0f;
    red[warp][g + 8][t] = have ? acc[ng < NG ? ng : 0][2] : 0.0f;
    red[warp][g + 8][t + 1] = have ? acc[ng < NG ? ng : 0][3] : 0.0f;
  }
  __syncthreads();
  // one output per thread: rank row tid / 16, token tid % 16
  const int jr = tid >> 4, t = tid & 15;
  if (t < M && j0 + jr < r) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kLoraDownThreads / 32; ++w) v += red[w][jr][t];
    v *= t_scale;  // 1, or 1 / (1 - p) when the input rows were dropped out
    const int64_t o = (int64_t)t * r + j0 + jr;
    sT[o] = __float2bfloat16_rn(v * s);
    if (T_hi) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      T_hi[o] = h;
      T_lo[o] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// s T for per-token adapters (multi-adapter decode): row k = t * r + j of s T
// is s_t * (X_t . A_t[j]) with token t's own adapter.  One warp per row: all of
// a round's sixteen 16-byte loads of A's row are issued before its products (X
// is read through L1, shared by the warps on the same token), then a butterfly
// sum.  The launcher sizes the grid to the SMs the decode GEMV that follows
// leaves free, so that this kernel runs beside it (programmatic dependent
// launch) instead of delaying its CTAs.
constexpr int kLoraDownMultiThreads = 512;
__global__ void __launch_bounds__(kLoraDownMultiThreads, 1) lora_down_multi_kernel(
    const __nv_bfloat16 *__restrict__ X, const MultiLora ml, int M, int64_t K, int r, __nv_bfloat16 *__restrict__ sT) {
  griddep_launch_dependents();
  constexpr int kWarps = kLoraDownMultiThreads / 32, U = 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows = M * r;
  const int64_t n16 = K / 8;  // 16-byte pieces per row (a multiple of 32)
  for (int k = blockIdx.x * kWarps + warp; k < rows; k += gridDim.x * kWarps) {
    const int t = k / r, j = k - t * r;
    const uint4 *arow = reinterpret_cast<const uint4 *>(ml.A[t] + (int64_t)j * K);
    const uint4 *xrow = reinterpret_cast<const uint4 *>(X + (int64_t)t * K);
    float acc = 0.0f;
    for (int64_t c0 = lane; c0 < n16; c0 += 32 * U) {
      uint4 av[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t c = c0 + 32 * u;
        av[u] = c < n16 ? __ldg(arow + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t c = c0 + 32 * u;
        const uint4 xv = c < n16 ? __ldg(xrow + c) : make_uint4(0, 0, 0, 0);
        const uint32_t aw[4] = {av[u].x, av[u].y, av[u].z, av[u].w};
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(bf16lo_to_f32(aw[e]), bf16lo_to_f32(xw[e]), acc);
          acc = fmaf(bf16hi_to_f32(aw[e]), bf16hi_to_f32(xw[e]), acc);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) sT[k] = __float2bfloat16_rn(acc * ml.s[t]);
  }
}

// LoRA term of the multi-adapter decode as its own pass over all SMs, after the
// GEMV has written the base product Yb (float32 [M, N]) to the workspace:
//   Y[t, n] = round(Yb[t, n] + sum_j B_t[n, j] (s T)[t, j]).
// For ranks with P = r / 8 a power of two: a warp reads 32 consecutive 16-byte
// pieces of B_t (32 / P rows, coalesced), each lane dots its piece with its
// slice of s T (kept in registers), the P lanes of a row combine their partials
// by a butterfly in fixed order and the first writes the row.  B is an input of
// the call, so each CTA loads its pieces before waiting for the GEMV
// (programmatic dependent launch) and overlaps the GEMV's tail where it can.
constexpr int kLoraUpThreads = 256, kLoraUpRounds = 4;
__global__ void __launch_bounds__(kLoraUpThreads) lora_up_multi_kernel(const float *__restrict__ Yb, const MultiLora ml,
                                                                      const __nv_bfloat16 *__restrict__ sT, int64_t N,
                                                                      int r, void *Y, int y_f32) {
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.y;
  const int P = r / 8, lgP = __ffs(P) - 1, rpw = 32 >> lgP;  // rows per warp round
  const int ch = lane & (P - 1);
  const int64_t rows_per_cta = (int64_t)(kLoraUpThreads / 32) * rpw * kLoraUpRounds;
  const int64_t row0 = blockIdx.x * rows_per_cta + (int64_t)warp * rpw * kLoraUpRounds + (lane >> lgP);
  const uint4 *B = reinterpret_cast<const uint4 *>(ml.B[t]);
  uint4 bv[kLoraUpRounds];
#pragma unroll
  for (int u = 0; u < kLoraUpRounds; ++u) {
    const int64_t n = row0 + u * rpw;
    bv[u] = n < N ? __ldg(B + n * P + ch) : make_uint4(0, 0, 0, 0);
  }
  ptx::griddep_wait();  // s T and Yb are complete
  const uint4 sv = __ldcg(reinterpret_cast<const uint4 *>(sT + (int64_t)t * r) + ch);
  const float s8[8] = {bf16lo_to_f32(sv.x), bf16hi_to_f32(sv.x), bf16lo_to_f32(sv.y), bf16hi_to_f32(sv.y),
                       bf16lo_to_f32(sv.z), bf16hi_to_f32(sv.z), bf16lo_to_f32(sv.w), bf16hi_to_f32(sv.w)};
#pragma unroll
  for (int u = 0; u < kLoraUpRounds; ++u) {
    const int64_t n = row0 + u * rpw;
    const uint32_t bw[4] = {bv[u].x, bv[u].y, bv[u].z, bv[u].w};
    float v = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v = fmaf(bf16lo_to_f32(bw[e]), s8[2 * e], v);
      v = fmaf(bf16hi_to_f32(bw[e]), s8[2 * e + 1], v);
    }
    for (int o = 1; o < P; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (ch == 0 && n < N) {
      const int64_t i = (int64_t)t * N + n;
      const float y = __ldcg(Yb + i) + v;
      if (y_f32) reinterpret_cast<float *>(Y)[i] = y;
      else reinterpret_cast<__nv_bfloat16 *>(Y)[i] = __float2bfloat16_rn(y);
    }
  }
}

// CTAs of the decode GEMV for N rows on `sms` SMs (as launch_gemv sizes it).
inline int gemv_grid_ctas(int64_t N, int sms, bool bulk) {
  const int num_rg = static_cast<int>((N + 15) / 16);
  const int cap = bulk ? kBulkMaxRG : kGemvMaxRG;
  int per = (num_rg + sms - 1) / sms;
  if (per > cap) per = cap;
  return (num_rg + per - 1) / per;
}

// Start of the dynamic shared-memory window of a kernel without static shared
// memory: after the block's system reservation.  The bulk kernel recomputes its
// layout from its real window start and reports an error if it does not fit.
inline uint32_t dyn_smem_base(int dev) {
  static std::once_flag flags[64];
  static uint32_t base[64];
  std::call_once(flags[dev], [&] {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
      v = 0;
      cudaGetLastError();
    }
    base[dev] = static_cast<uint32_t>(v);
  });
  return base[dev];
}

inline qlora_status launch_gemv(GemvArgs g, const CUtensorMap *tm_codes, int dev, int sms, cudaStream_t st) {
  const int num_rg = static_cast<int>((g.N + 15) / 16);
  bool bulk = tm_codes != nullptr && gemv_bulk_ok(g.N, g.K);
  const int cap = bulk ? kBulkMaxRG : kGemvMaxRG;
  int per = (num_rg + sms - 1) / sms;
  if (per > cap) per = cap;
  g.rg_per_cta = per;
  g.stages = 0;
  int smem = 0;
  if (bulk) {
    const int64_t CH = g.K < 4096 ? g.K : 4096;
    const uint32_t base = dyn_smem_base(dev);
    g.stages = gemv_bulk_stages(g.K, g.M, base, per * static_cast<int>(g.K / CH));
    if (g.stages == 0) bulk = false;
    else {
      smem = gemv_bulk_smem_bytes(g.K, g.stages, g.M, base);
      g.lay = gemv_bulk_layout(base, gemv_bulk_stage_bytes(g.K), g.stages, gemv_bulk_red_bytes(g.M));
      g.lay_base = base;
    }
  }
  if (!bulk && g.multi) return QLORA_ERR_UNSUPPORTED_SHAPE;  // per-token adapters: staged kernel only
  if (!bulk) {
    per = (num_rg + sms - 1) / sms;
    if (per > kGemvMaxRG) per = kGemvMaxRG;
    g.rg_per_cta = per;
    smem = 256 * 32 * 4 + per * kGemvWarps * 256 * 4;
  }
  const int grid = (num_rg + per - 1) / per;
  static std::once_flag flags[4][64];
  static qlora_status results[4][64];
  const bool two = g.M > 8;
  const int which = (bulk ? 2 : 0) + (two ? 1 : 0);
  const int max_smem = bulk ? static_cast<int>(kBulkSmemLimit) : 256 * 32 * 4 + kGemvMaxRG * kGemvWarps * 256 * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (bulk) {
    auto kernel = two ? nf4_gemv_bulk_kernel<2> : nf4_gemv_bulk_kernel<1>;
    std::call_once(flags[which][dev], [&] {
      results[which][dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) ==
                                    cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
      cudaGetLastError();
    });
    if (results[which][dev] != QLORA_OK) return results[which][dev];
    e = cudaLaunchKernelEx(&cfg, kernel, *tm_codes, g, smem);
  } else {
    auto kernel = two ? nf4_gemv_lora_kernel<2> : nf4_gemv_lora_kernel<1>;
    std::call_once(flags[which][dev], [&] {
      results[which][dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) ==
                                    cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
      cudaGetLastError();
    });
    if (results[which][dev] != QLORA_OK) return results[which][dev];
    e = cudaLaunchKernelEx(&cfg, kernel, g);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

}  // namespace qlora
