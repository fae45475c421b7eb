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

#include "gemm_kernel.cuh"
#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

// ---------------------------------------------------------------------------
// Merged export on the tensor cores (tcgen05, accumulators in TMEM).  Persistent
// CTAs walk the 128-row x 256-column tiles of W_merged.  Per tile:
//   * warp 0 (one thread) loads by TMA, per 64 ranks, B's 128 rows (K-major)
//     and A's 64 x 256 block (MN-major); warp 2 (one thread) loads the tile's
//     NF4 codes (128 rows x 128 bytes, 128-byte swizzle) up to four tiles ahead;
//   * warp 1 (one thread) issues tcgen05.mma M = 128, N = 256, K = 16 into one
//     of two TMEM accumulators: (B A)[n0.., k0..] in float32;
//   * warps 4..19 (TMEM lane quadrant warp % 4, 64-column quarter (warp - 4) / 4
//     of the tile) read accumulator rows with tcgen05.ld, decode W' from the
//     codes and the block scale, form fma(s, (B A), W') in float32, round once
//     to bf16 and write the tile through a swizzled shared-memory buffer that a
//     TMA store copies out (clipped at the matrix edge).  Sixteen epilogue warps
//     (four per scheduler) keep the decode, which is the longest step, fed.
// Loads, products, the epilogue and the stores of consecutive tiles overlap.
// HBM traffic per weight: 0.5 B of code + 1/64 B of scale + 2 B written; the
// adapter's tiles come from L2.  Every wait is bounded; one that gives up
// records QLORA_ERR_TIMEOUT in the status word, the other roles leave, copies
// and products in flight are drained and TMEM is freed.
// ---------------------------------------------------------------------------
constexpr int kMergeBM = 128;
constexpr int kMergeBN = 256;
constexpr int kMergeThreads = 640;
constexpr int kMergeEpiWarps = 16;
constexpr int kMergeSAB = 2;  // stages of (B rows, A block) per 64 ranks
constexpr int kMergeSC = 4;   // stages of codes
constexpr uint32_t kMergeAStage = kMergeBM * 64 * 2;  // B rows: 128 x 64 ranks
constexpr uint32_t kMergeBStage = 64 * kMergeBN * 2;  // A block: 64 ranks x 256 columns
constexpr uint32_t kMergeABStage = kMergeAStage + kMergeBStage;
constexpr uint32_t kMergeCStage = kMergeBM * 128;  // codes: 128 rows x 256 columns / 2
constexpr uint32_t kMergeOutBuf = 32 * 128;         // 32 rows x 64 columns of bf16
constexpr uint32_t kMergeOutBytes = kMergeEpiWarps * kMergeOutBuf;
constexpr uint32_t kMergeSmemBytes =
    kMergeSAB * kMergeABStage + kMergeSC * kMergeCStage + kMergeOutBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kMergeTmemCols = 2 * kMergeBN;
constexpr uint32_t kMergeIdesc = ptx::idesc_bf16(kMergeBM, kMergeBN, 0, 1);
static_assert(kMergeSmemBytes <= 227 * 1024, "shared memory");

struct MergeArgs {
  const uint8_t *scale_codes;
  const float *c2;
  int64_t N, K;
  int r;
  float s;  // alpha / r
  int fmt;  // qlora_scale_format
  uint32_t *status;
};

__global__ void __launch_bounds__(kMergeThreads, 1)
    nf4_lora_merge_kernel(const __grid_constant__ CUtensorMap tmCodes, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmOut,
                          const MergeArgs a) {
  extern __shared__ uint8_t merge_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(merge_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sAB = smem;
  uint8_t *sC = sAB + kMergeSAB * kMergeABStage;
  uint8_t *sOut = sC + kMergeSC * kMergeCStage;
  uint64_t *full_ab = reinterpret_cast<uint64_t *>(sOut + kMergeOutBytes);
  uint64_t *empty_ab = full_ab + kMergeSAB;
  uint64_t *full_c = empty_ab + kMergeSAB;
  uint64_t *empty_c = full_c + kMergeSC;
  uint64_t *acc_full = empty_c + kMergeSC;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMergeSAB; ++i) { ptx::mbar_init(&full_ab[i], 1); ptx::mbar_init(&empty_ab[i], 1); }
    for (int i = 0; i < kMergeSC; ++i) {
      ptx::mbar_init(&full_c[i], 1);
      ptx::mbar_init(&empty_c[i], kMergeEpiWarps);
    }
    for (int i = 0; i < 2; ++i) { ptx::mbar_init(&acc_full[i], 1); ptx::mbar_init(&acc_empty[i], kMergeEpiWarps); }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmCodes);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmOut);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kMergeTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t N = a.N, K = a.K;
  // tile t = row block rb * ncol + column block cb (fewer than 2^31 tiles); a
  // CTA's tiles t, t + G, ... are walked by steps of (G / ncol, G % ncol)
  const int ncol = static_cast<int>((K + kMergeBN - 1) / kMergeBN);
  const int tiles = static_cast<int>((N + kMergeBM - 1) / kMergeBM) * ncol;
  const int G = gridDim.x, step_r = G / ncol, step_c = G - step_r * ncol;
  const int rsteps = (a.r + 63) / 64;
  struct TilePos {
    int t, rb, cb;
  };
  auto first_tile = [&]() {
    const int t = blockIdx.x, rb = t / ncol;
    return TilePos{t, rb, t - rb * ncol};
  };
  auto next_tile = [&](TilePos &p) {
    p.t += G;
    p.rb += step_r;
    p.cb += step_c;
    if (p.cb >= ncol) {
      p.cb -= ncol;
      ++p.rb;
    }
  };
  auto fail = [&]() {
    raise_status(a.status, QLORA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer: adapter tiles
    if (ptx::elect_one()) {
      uint32_t sab = 0, pab = 0;
      int issued_ab = 0;
      bool ok = true;
      for (TilePos p = first_tile(); p.t < tiles && ok; next_tile(p)) {
        const int64_t n0 = static_cast<int64_t>(p.rb) * kMergeBM, k0 = static_cast<int64_t>(p.cb) * kMergeBN;
        for (int j = 0; j < rsteps; ++j) {
          if (!ptx::mbar_wait(&empty_ab[sab], pab ^ 1, abort_flag)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&full_ab[sab], kMergeABStage);
          uint8_t *d = sAB + sab * kMergeABStage;
          ptx::tma_load_2d(d, &tmB, &full_ab[sab], 64 * j, static_cast<int32_t>(n0));
          for (int u = 0; u < kMergeBN / 64; ++u)
            ptx::tma_load_2d(d + kMergeAStage + u * 8192, &tmA, &full_ab[sab], static_cast<int32_t>(k0 + 64 * u),
                             64 * j);
          ++issued_ab;
          if (++sab == kMergeSAB) { sab = 0; pab ^= 1; }
        }
      }
      if (!ok) fail();
      // the last (up to) kMergeSAB copies must land before the CTA exits
      for (int i = 0; i < kMergeSAB && i < issued_ab; ++i) {
        if (sab == 0) { sab = kMergeSAB - 1; pab ^= 1; } else { --sab; }
        ptx::mbar_wait(&full_ab[sab], pab, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ TMA producer: codes
    if (ptx::elect_one()) {
      uint32_t sc = 0, pc = 0;
      int issued_c = 0;
      bool ok = true;
      for (TilePos p = first_tile(); p.t < tiles; next_tile(p)) {
        const int64_t n0 = static_cast<int64_t>(p.rb) * kMergeBM, k0 = static_cast<int64_t>(p.cb) * kMergeBN;
        if (!ptx::mbar_wait(&empty_c[sc], pc ^ 1, abort_flag)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&full_c[sc], kMergeCStage);
        ptx::tma_load_2d(sC + sc * kMergeCStage, &tmCodes, &full_c[sc], static_cast<int32_t>(k0 / 2),
                         static_cast<int32_t>(n0));
        ++issued_c;
        if (++sc == kMergeSC) { sc = 0; pc ^= 1; }
      }
      if (!ok) fail();
      for (int i = 0; i < kMergeSC && i < issued_c; ++i) {
        if (sc == 0) { sc = kMergeSC - 1; pc ^= 1; } else { --sc; }
        ptx::mbar_wait(&full_c[sc], pc, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (ptx::elect_one()) {
      uint32_t sab = 0, pab = 0;
      int it = 0;
      bool ok = true;
      const uint32_t sAB0 = ptx::smem_addr(sAB);
      for (int t = blockIdx.x; t < tiles && ok; t += G, ++it) {
        const int acc = it & 1;
        if (!ptx::mbar_wait(&acc_empty[acc], ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kMergeBN;
        for (int j = 0; j < rsteps; ++j) {
          if (!ptx::mbar_wait(&full_ab[sab], pab, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a_base = sAB0 + sab * kMergeABStage, b_base = a_base + kMergeAStage;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            ptx::mma_bf16(d_tmem, ptx::smem_desc_sw128(a_base + k16 * 32, 16, 1024),
                          ptx::smem_desc_sw128(b_base + k16 * 2048, 8192, 1024), kMergeIdesc, (j | k16) ? 1u : 0u);
          ptx::mma_commit(&empty_ab[sab]);
          if (++sab == kMergeSAB) { sab = 0; pab ^= 1; }
        }
        if (ok) ptx::mma_commit(&acc_full[acc]);
      }
      if (!ok) fail();
      ptx::mma_commit(drain);  // every product issued has completed
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 4, qd = warp & 3, cq = e >> 2;
    const int row_t = qd * 32 + lane;  // tile row of this thread (TMEM lane)
    uint8_t *buf = sOut + e * kMergeOutBuf;
    const int64_t nbk = K / 64;
    // scale code and second-level constant of this thread's row in its 64-column
    // block of tile t: loaded one tile ahead (the raw values, so that nothing
    // waits for the loads until the tile that uses them)
    auto scale_src = [&](const TilePos &p, uint32_t &qv, float &cv) {
      qv = 0u;
      cv = 0.0f;
      if (p.t >= tiles) return;
      const int64_t n = static_cast<int64_t>(p.rb) * kMergeBM + row_t, kb = static_cast<int64_t>(p.cb) * 4 + cq;
      if (n < N && kb < nbk) {
        const int64_t b = n * nbk + kb;
        qv = __ldg(a.scale_codes + b);
        cv = __ldg(a.c2 + (b >> 8));
      }
    };
    uint32_t qv;
    float cv;
    TilePos ahead = first_tile();  // the tile whose scale is loaded next
    scale_src(ahead, qv, cv);
    uint32_t sc = 0, pc = 0;
    int it = 0;
    for (TilePos p = first_tile(); p.t < tiles; next_tile(p), ++it) {
      const int64_t n0 = static_cast<int64_t>(p.rb) * kMergeBM, k0 = static_cast<int64_t>(p.cb) * kMergeBN;
      const float S = __fmul_rn(scale_code_value(qv, a.fmt), cv);  // S' = fl32(code value * c2)
      next_tile(ahead);
      scale_src(ahead, qv, cv);
      const int acc = it & 1;
      const bool ready = ptx::mbar_wait(&full_c[sc], pc, abort_flag) &&
                         ptx::mbar_wait(&acc_full[acc], (it >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ready)) {  // the warp leaves together (its TMEM loads are warp-wide)
        if (lane == 0) fail();
        break;
      }
      ptx::tc_fence_after();
      // codes of columns 64 cq .. +63 of the row: 16-byte chunks 2 cq, 2 cq + 1
      const uint8_t *crow = sC + sc * kMergeCStage + row_t * 128;
      const uint4 c0 = *reinterpret_cast<const uint4 *>(crow + (((2 * cq) ^ (row_t & 7)) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4 *>(crow + (((2 * cq + 1) ^ (row_t & 7)) << 4));
      uint32_t lo[4], hi[4];
      nf4_planes(S, lo, hi);
      const uint32_t tcol = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + acc * kMergeBN + cq * 64;
      // the store that last read the buffer (one tile back) has finished reading it
      if (lane == 0) ptx::bulk_wait_read0();
      __syncwarp();
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {  // 32 columns at a time
        uint32_t v[32];
        ptx::tmem_ld32(tcol + 32 * qi, v);
        const uint32_t cw[4] = {qi ? c1.x : c0.x, qi ? c1.y : c0.y, qi ? c1.z : c0.z, qi ? c1.w : c0.w};
        uint32_t w[16];  // W' of columns 32 qi + 2i, + 1 (bf16 pairs)
#pragma unroll
        for (int j = 0; j < 4; ++j) nf4_word(cw[j], lo, hi, w + 4 * j);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 8 columns per 16-byte chunk
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t wp = w[4 * c + i];
            pk[i] = pack_bf16x2(__fmaf_rn(a.s, __uint_as_float(v[8 * c + 2 * i]), bf16lo_to_f32(wp)),
                                __fmaf_rn(a.s, __uint_as_float(v[8 * c + 2 * i + 1]), bf16hi_to_f32(wp)));
          }
          const int chunk = 4 * qi + c;
          *reinterpret_cast<uint4 *>(buf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      // this tile's codes and accumulator are read
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&empty_c[sc]);
        ptx::mbar_arrive(&acc_empty[acc]);
        const int64_t x = k0 + cq * 64, y = n0 + qd * 32;
        if (x < K && y < N) {
          ptx::tma_store_2d(&tmOut, buf, static_cast<int32_t>(x), static_cast<int32_t>(y));
          ptx::bulk_commit();
        }
      }
      if (++sc == kMergeSC) { sc = 0; pc ^= 1; }
    }
    if (lane == 0) ptx::bulk_wait_all();  // the stores have completed
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kMergeTmemCols);
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
