// The steps after the backward pass on the adapters:
//
// * Merged export, W_merged = bf16_rne(W' + s B A): "QLoRA" (Ultralytics
//   glossary), "Trade-offs": merging the adapters into the base model first
//   needs it dequantised to 16 bit; "What is LoRA?" (IBM): the trained
//   low-rank update merges into the frozen weights for deployment.
// * AdamW step on the adapter parameters: "Grokking QLoRA" (vnread), "Paged
//   Optimizers": Adam keeps a momentum and a variance per trained parameter;
//   the update is decoupled-weight-decay Adam with bias correction.
#pragma once

#include "nf4_device.cuh"

namespace qlora {

// ---------------------------------------------------------------------------
// Merged export.  One CTA (8 warps) makes kMergePasses consecutive 128 x 128
// tiles of one 128-row block of W_merged: the low-rank product s B A on
// mma.sync tensor cores (bf16 in, fp32 accumulate) from shared-memory copies of
// B's 128 rows (staged once per CTA) and of A's columns of the tile (both
// row-major, rows padded by 16 bytes so ldmatrix reads are conflict-free; A's
// fragments come transposed by ldmatrix.trans); W' decoded from the tile's
// codes and block scales staged in shared memory; the sum in fp32, rounded to
// bf16 once, staged in shared memory and stored with 16-byte writes.  For ranks
// up to 64 the next tile's A columns, codes and scales are loaded into
// registers while the current tile is computed and stored.
// HBM traffic per weight: 0.5 B of code + 1/64 B of scale + 2 B written.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 256;
constexpr int kMergeTile = 128;
constexpr int kMergeMaxK16 = 16;  // r <= 256
constexpr int kMergePasses = 4;   // column tiles per CTA
constexpr int kMergePreR16 = 64;  // ranks whose next A tile fits the prefetch registers

__host__ __device__ inline int merge_r16(int r) { return ((r + 15) / 16) * 16; }
__host__ __device__ inline size_t merge_operand_bytes(int r) {
  return static_cast<size_t>(kMergeTile) * (merge_r16(r) + 8) * 2        // B rows [128][r16 + 8]
         + static_cast<size_t>(merge_r16(r)) * (kMergeTile + 8) * 2;     // A tile [r16][136]
}
inline size_t merge_smem_bytes(int r) {
  const size_t outb = static_cast<size_t>(kMergeTile) * (kMergeTile + 8) * 2;  // bf16 [128][136]
  return merge_operand_bytes(r) + outb + kMergeTile * 64 + kMergeTile * 2 * 4 + 16 * 4;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t &b0, uint32_t &b1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(addr));
}

__global__ void __launch_bounds__(kMergeThreads, 2) nf4_lora_merge_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale_codes, const float *__restrict__ c2,
    int64_t N, int64_t K, const __nv_bfloat16 *__restrict__ A, const __nv_bfloat16 *__restrict__ B, int r, float s,
    __nv_bfloat16 *__restrict__ out, int fmt) {
  extern __shared__ __align__(16) uint8_t merge_smem[];
  const int r16 = merge_r16(r), ldb = r16 + 8;
  constexpr int LDA = kMergeTile + 8, LDO = kMergeTile + 8;
  __nv_bfloat16 *sB = reinterpret_cast<__nv_bfloat16 *>(merge_smem);  // [128][ldb]: B rows n0..
  __nv_bfloat16 *sA = sB + kMergeTile * ldb;                         // [r16][LDA]: A columns k0..
  __nv_bfloat16 *sOut = sA + r16 * LDA;                              // [128][LDO]
  uint8_t *sCodes = reinterpret_cast<uint8_t *>(sOut + kMergeTile * LDO);  // [128][64]
  float *sS = reinterpret_cast<float *>(sCodes + kMergeTile * 64);         // [128][2]
  float *sLv = sS + kMergeTile * 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t n0 = (int64_t)blockIdx.y * kMergeTile;
  const int64_t kt0 = (int64_t)blockIdx.x * kMergePasses;           // first column tile of this CTA
  const int64_t ktiles = (K + kMergeTile - 1) / kMergeTile;
  const int passes = static_cast<int>(ktiles - kt0 < kMergePasses ? ktiles - kt0 : kMergePasses);
  const int64_t nbk = K / 64;
  const bool pre = r16 <= kMergePreR16;

  if (tid < 16) sLv[tid] = __uint_as_float(kNf4LevelBits[tid]);
  for (int i = tid; i < kMergeTile * (r16 / 8); i += kMergeThreads) {  // B rows (zero past N and r)
    const int row = i / (r16 / 8), c8 = (i % (r16 / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n0 + row < N && c8 < r) v = __ldg(reinterpret_cast<const uint4 *>(B + (n0 + row) * r + c8));
    *reinterpret_cast<uint4 *>(sB + row * ldb + c8) = v;
  }

  // One tile's A columns, codes and block scales: loaded into registers
  // (ranks <= 64) and stored to shared memory when its space is free.
  uint4 pa[kMergePreR16 / 16];  // A: r16 x 128 bf16 = 16 r16 bytes, 16 bytes per thread per 16 ranks
  uint4 pc[2];                  // codes: 128 rows x 64 bytes, 32 bytes per thread
  float ps;                     // block scale of (row tid / 2, block tid % 2)
  auto load_tile = [&](int64_t kt) {
    const int64_t k0 = kt * kMergeTile;
    const int kcols = static_cast<int>(K - k0 < kMergeTile ? K - k0 : kMergeTile);
#pragma unroll
    for (int u = 0; u < kMergePreR16 / 16; ++u) {
      const int i = tid + u * kMergeThreads;  // 16-byte piece i of the A tile
      const int j = i / (kMergeTile / 8), c8 = (i % (kMergeTile / 8)) * 8;
      pa[u] = make_uint4(0, 0, 0, 0);
      if (j < r16 && j < r && c8 < kcols) pa[u] = __ldg(reinterpret_cast<const uint4 *>(A + (int64_t)j * K + k0 + c8));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = tid + u * kMergeThreads;
      const int row = i >> 2, c16 = (i & 3) * 16;
      pc[u] = make_uint4(0, 0, 0, 0);
      if (n0 + row < N && 2 * c16 < kcols)
        pc[u] = __ldg(reinterpret_cast<const uint4 *>(codes + (n0 + row) * (K / 2) + k0 / 2 + c16));
    }
    const int row = tid >> 1, b = tid & 1;
    ps = 0.0f;
    if (n0 + row < N && 64 * b < kcols) ps = block_scale(scale_codes, c2, (n0 + row) * nbk + k0 / 64 + b, fmt);
  };
  auto store_tile = [&]() {
#pragma unroll
    for (int u = 0; u < kMergePreR16 / 16; ++u) {
      const int i = tid + u * kMergeThreads;
      const int j = i / (kMergeTile / 8), c8 = (i % (kMergeTile / 8)) * 8;
      if (j < r16) *reinterpret_cast<uint4 *>(sA + j * LDA + c8) = pa[u];
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = tid + u * kMergeThreads;
      *reinterpret_cast<uint4 *>(sCodes + (i >> 2) * 64 + (i & 3) * 16) = pc[u];
    }
    sS[tid] = ps;
  };
  // ranks above 64: the A tile straight to shared memory (no prefetch)
  auto direct_a = [&](int64_t kt) {
    const int64_t k0 = kt * kMergeTile;
    const int kcols = static_cast<int>(K - k0 < kMergeTile ? K - k0 : kMergeTile);
    for (int i = tid; i < r16 * (kMergeTile / 8); i += kMergeThreads) {
      const int j = i / (kMergeTile / 8), c8 = (i % (kMergeTile / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j < r && c8 < kcols) v = __ldg(reinterpret_cast<const uint4 *>(A + (int64_t)j * K + k0 + c8));
      *reinterpret_cast<uint4 *>(sA + j * LDA + c8) = v;
    }
  };

  load_tile(kt0);
  store_tile();
  if (!pre) direct_a(kt0);
  __syncthreads();

  const uint32_t sB0 = static_cast<uint32_t>(__cvta_generic_to_shared(sB));
  const uint32_t sA0 = static_cast<uint32_t>(__cvta_generic_to_shared(sA));
  // A-fragment rows: lanes 0-15 rows 0..15 at column kk, lanes 16-31 the same rows at kk + 8
  const uint32_t a_row = static_cast<uint32_t>(warp * 16 + (lane & 15));
  const uint32_t a_col = static_cast<uint32_t>((lane >> 4) * 8);
  for (int p = 0; p < passes; ++p) {
    const int64_t k0 = (kt0 + p) * kMergeTile;
    const int kcols = static_cast<int>(K - k0 < kMergeTile ? K - k0 : kMergeTile);
    if (p + 1 < passes) load_tile(kt0 + p + 1);  // in flight during this tile's work

    // warp w: rows [16w, 16w + 16) of the tile, all 128 columns (16 n8 tiles)
    float acc[kMergeTile / 8][4];
#pragma unroll
    for (int t = 0; t < kMergeTile / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
#pragma unroll
    for (int k16 = 0; k16 < kMergeMaxK16; ++k16) {
      if (16 * k16 >= r16) break;
      uint32_t af[4];
      ldmatrix_x4(af, sB0 + (a_row * ldb + 16 * k16 + a_col) * 2);
      // B fragments: lanes 0-15 give rows kk + (lane & 15) of A's tile at column 8t
      const uint32_t b_row = sA0 + ((16 * k16 + (lane & 15)) * LDA) * 2;
#pragma unroll
      for (int t = 0; t < kMergeTile / 8; ++t) {
        uint32_t b0, b1;
        ldmatrix_x2_trans(b0, b1, b_row + t * 16);
        mma_bf16_16816(acc[t], af[0], af[1], af[2], af[3], b0, b1);
      }
    }
    const int r0 = warp * 16 + g, r1 = r0 + 8;
#pragma unroll
    for (int t = 0; t < kMergeTile / 8; ++t) {
      const int c = t * 8 + 2 * q;  // C fragment: rows r0 / r1, columns c, c + 1
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = h ? r1 : r0;
        const uint8_t byte = sCodes[row * 64 + (c >> 1)];
        const float S = sS[row * 2 + (c >> 6)];
        const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sLv[byte & 15], S)));
        const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sLv[byte >> 4], S)));
        const float v0 = __fmaf_rn(s, acc[t][2 * h], w0), v1 = __fmaf_rn(s, acc[t][2 * h + 1], w1);
        *reinterpret_cast<uint32_t *>(sOut + row * LDO + c) = pack_bf16x2(v0, v1);
      }
    }
    __syncthreads();  // the tile is in sOut; sA, sCodes and sS are read
    for (int i = tid; i < kMergeTile * (kMergeTile / 8); i += kMergeThreads) {
      const int row = i / (kMergeTile / 8), c8 = (i % (kMergeTile / 8)) * 8;
      if (n0 + row < N && c8 < kcols)
        *reinterpret_cast<uint4 *>(out + (n0 + row) * K + k0 + c8) =
            *reinterpret_cast<const uint4 *>(sOut + row * LDO + c8);
    }
    if (p + 1 < passes) {
      store_tile();
      if (!pre) direct_a(kt0 + p + 1);
    }
    __syncthreads();  // the next tile is staged; sOut is stored
  }
}

// ---------------------------------------------------------------------------
// LoRA dropout input: Xm = X * keep (bf16, exact: each element is X or 0), keep
// packed one bit per element (bit k % 8 of byte k / 8 of each row).  The
// 1 / (1 - p) factor is applied to the products computed from Xm.  One thread
// per 8 elements (16 bytes of X, one mask byte).
// ---------------------------------------------------------------------------
__global__ void keep_mask_kernel(const __nv_bfloat16 *__restrict__ X, const uint8_t *__restrict__ keep,
                                 int64_t n8, __nv_bfloat16 *__restrict__ Xm) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t b = keep[i];
    uint4 v = __ldg(reinterpret_cast<const uint4 *>(X) + i);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = (b >> (2 * e)) & 1u ? 0x0000ffffu : 0u, hi = (b >> (2 * e + 1)) & 1u ? 0xffff0000u : 0u;
      w[e] &= lo | hi;
    }
    reinterpret_cast<uint4 *>(Xm)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// AdamW on flat float32 arrays (parameters, gradients, momentum, variance), in
// the order of the definition:
//   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2;
//   p = p (1 - lr wd) - (lr / bc1) m / (sqrt(v) / sqrt(bc2) + eps)
// with bc1 = 1 - b1^t, bc2 = 1 - b2^t from the host; optionally writes the bf16
// copy the layer reads.  HBM traffic per parameter: 16 B read, 12 B written
// (+2 B for the bf16 copy).
// ---------------------------------------------------------------------------
struct AdamWConsts {
  float lr, beta1, beta2, eps, decay_factor, step_size, sqrt_bc2;
};

__device__ __forceinline__ void adamw_one(float &p, float g, float &m, float &v, const AdamWConsts &c) {
  m = __fadd_rn(__fmul_rn(c.beta1, m), __fmul_rn(1.0f - c.beta1, g));
  v = __fadd_rn(__fmul_rn(c.beta2, v), __fmul_rn(1.0f - c.beta2, __fmul_rn(g, g)));
  const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(v), c.sqrt_bc2), c.eps);
  p = __fsub_rn(__fmul_rn(p, c.decay_factor), __fdiv_rn(__fmul_rn(c.step_size, m), denom));
}

__global__ void adamw_kernel(float *__restrict__ p, __nv_bfloat16 *__restrict__ p16, const float *__restrict__ g,
                             float *__restrict__ m, float *__restrict__ v, int64_t n, AdamWConsts c) {
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pp = reinterpret_cast<float4 *>(p)[i];
    const float4 gg = reinterpret_cast<const float4 *>(g)[i];
    float4 mm = reinterpret_cast<float4 *>(m)[i];
    float4 vv = reinterpret_cast<float4 *>(v)[i];
    adamw_one(pp.x, gg.x, mm.x, vv.x, c);
    adamw_one(pp.y, gg.y, mm.y, vv.y, c);
    adamw_one(pp.z, gg.z, mm.z, vv.z, c);
    adamw_one(pp.w, gg.w, mm.w, vv.w, c);
    reinterpret_cast<float4 *>(p)[i] = pp;
    reinterpret_cast<float4 *>(m)[i] = mm;
    reinterpret_cast<float4 *>(v)[i] = vv;
    if (p16) reinterpret_cast<uint2 *>(p16)[i] = make_uint2(pack_bf16x2(pp.x, pp.y), pack_bf16x2(pp.z, pp.w));
  }
  for (int64_t i = 4 * n4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) {
    float pp = p[i], mm = m[i], vv = v[i];
    adamw_one(pp, g[i], mm, vv, c);
    p[i] = pp;
    m[i] = mm;
    v[i] = vv;
    if (p16) p16[i] = __float2bfloat16_rn(pp);
  }
}

}  // namespace qlora
