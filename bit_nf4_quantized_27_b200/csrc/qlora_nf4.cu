// C ABI of the NF4 frozen-linear + LoRA library (see include/qlora_nf4.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "gemm_kernel.cuh"
#include "gemm_pair_kernel.cuh"
#include "adapter_kernels.cuh"
#include "decode_kernel.cuh"
#include "gemv_kernel.cuh"
#include "host_common.h"
#include "qlora_nf4.h"
#include "quant_kernels.cuh"
#include "selftest_kernel.cuh"

using namespace qlora;

// Token subtiles of 128 per fused-GEMM tile: each decoded 256x64 W' tile feeds
// MT accumulators, so the decode work per tensor-core FLOP falls as 1/MT.
#ifndef QLORA_FUSED_MT
#define QLORA_FUSED_MT 2
#endif
constexpr int kFusedMT = QLORA_FUSED_MT;

namespace {
// Device address of the library status word on device `dev` (defined below).
qlora_status library_status_addr(int dev, uint32_t **out);

// ---------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime: no link-time
// dependency on libcuda).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] with row stride `ld` elements.
bool make_tmap(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, uint32_t esize, uint64_t inner,
               uint64_t outer, uint64_t ld, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  std::memset(m, 0, sizeof(*m));
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * esize};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// NF4 codes [N][K/2 bytes] as a 3-D map (128 bytes, N rows, K/256 chunks of 128
// bytes), box 128 x `rows` x `chunks`, 128-byte swizzle: the decode kernels'
// stage layout [chunk][row][128 B].
bool tmap_codes_gemv(CUtensorMap *m, const void *codes, int64_t N, int64_t K, uint32_t chunks, uint32_t rows = 16) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K / 256)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2), 128};
  const cuuint32_t box[3] = {128, rows, chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(codes), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// LoRA B [N, r] bf16 as a 3-D map (64 ranks, N rows, r/64 chunks of 128 bytes;
// for r <= 64 one chunk whose ranks past r read as zeros), box 64 x `rows` x
// chunks with the 128-byte swizzle: the decode kernel's per-unit B-row layout
// [chunk][row][128 B].
bool tmap_brows(CUtensorMap *m, const void *B, int64_t N, int r, uint32_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t chunks = r <= 64 ? 1u : static_cast<uint32_t>(r / 64);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(r <= 64 ? r : 64), static_cast<cuuint64_t>(N), chunks};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(r) * 2, 128};
  const cuuint32_t box[3] = {64, rows, chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(B), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool tmap_bf16(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
               uint32_t box_outer) {
  return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, inner, outer, inner, box_inner, box_outer, true);
}

// Launch with programmatic dependent launch allowed: the kernel's set-up
// overlaps the preceding kernel's tail, and the kernel waits for that kernel
// (griddepcontrol.wait) before it touches global memory.
template <typename... KArgs, typename... Args>
qlora_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

// Once per device and kernel: allow the kernel's dynamic shared memory.
template <typename F>
qlora_status set_smem(F kernel, int bytes, int dev, std::once_flag *flags, qlora_status *results) {
  std::call_once(flags[dev], [&] {
    results[dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
                       ? QLORA_OK
                       : QLORA_ERR_CUDA;
    cudaGetLastError();
  });
  return results[dev];
}

// The fused NF4 GEMM on CTA pairs, persistent over as many pairs as fit at
// once.  Returns QLORA_ERR_UNSUPPORTED_SHAPE when no pair cluster can be
// resident (the caller then uses the single-CTA kernel).
template <bool B_MN, int MT>
qlora_status launch_gemm_pair(const CUtensorMap &tmA, const CUtensorMap &tmA2, const CUtensorMap &tmCodes,
                              const GemmArgs &args, int dev, cudaStream_t st) {
  using C = GemmPairCfg<B_MN, MT>;
  auto kernel = gemm_nf4_pair_kernel<B_MN, MT>;
  static std::once_flag flags[64], occ_flags[64];
  static qlora_status results[64];
  static int max_clusters[64];
  qlora_status s = set_smem(kernel, C::SMEM_BYTES, dev, flags, results);
  if (s != QLORA_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the cluster shape alone for the occupancy query
  std::call_once(occ_flags[dev], [&] {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &q) != cudaSuccess) n = 0;
    cudaGetLastError();
    max_clusters[dev] = n;
  });
  if (max_clusters[dev] <= 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int num_m = (args.M_rows + 2 * C::BM * MT - 1) / (2 * C::BM * MT);
  const int num_n = (args.N_cols + C::BN - 1) / C::BN;
  const int clusters = std::max(1, std::min(num_m * num_n, max_clusters[dev]));
  cfg.gridDim = dim3(2 * clusters);
  cfg.numAttrs = 2;  // and programmatic dependent launch
  if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmA2, tmCodes, args) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

// Token counts from which the fused GEMMs run on CTA pairs (512-token tiles).
constexpr int64_t kPairMinRows = 257;

// One tcgen05 GEMM launch; with `group` (a second problem of the same tile shape,
// no K split, no LoRA steps, maps gA / gB / gB2) both problems share the launch
// and run at once.
template <bool A_MN, bool B_MN, bool NF4, int BN, int MT>
qlora_status launch_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmA2,
                         const CUtensorMap &tmB2, const CUtensorMap &tmCodes, const GemmArgs &args, int dev, int sms,
                         cudaStream_t st, const GemmArgs *group = nullptr, const CUtensorMap *gA = nullptr,
                         const CUtensorMap *gB = nullptr, const CUtensorMap *gB2 = nullptr) {
  using C = GemmCfg<A_MN, B_MN, NF4, BN, MT>;
  auto kernel = gemm_tc_kernel<A_MN, B_MN, NF4, BN, MT>;
  static std::once_flag flags[64];
  static qlora_status results[64];
  qlora_status s = set_smem(kernel, C::SMEM_BYTES, dev, flags, results);
  if (s != QLORA_OK) return s;
  const int tile_n = args.hilo_cols ? BN / 2 : BN;
  const int num_m = (args.M_rows + C::BM * MT - 1) / (C::BM * MT);
  const int num_n = (args.N_cols + tile_n - 1) / tile_n;
  int tiles = num_m * num_n * std::max(1, args.ksplit);
  GemmArgs none{};  // no second problem
  if (group) {
    if (NF4 || group->ksplit > 1 || group->lora_steps || group->hilo_cols != args.hilo_cols || group->M_rows <= 0)
      return QLORA_ERR_INVALID_ARGUMENT;
    tiles += ((group->M_rows + C::BM * MT - 1) / (C::BM * MT)) * ((group->N_cols + tile_n - 1) / tile_n);
  }
  const int grid = std::max(1, std::min(tiles, sms));
  return launch_pdl(kernel, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, tmA, tmB, tmA2, tmB2, tmCodes, args,
                    group ? *gA : tmA, group ? *gB : tmB, group ? *gB2 : tmB2, group ? *group : none);
}

uint32_t *status_ptr(void *ws) { return reinterpret_cast<uint32_t *>(ws); }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

qlora_status check_lora(const qlora_lora *ad) {
  if (!ad || !ad->A || !ad->B) return QLORA_ERR_INVALID_ARGUMENT;
  if (ad->r < 8 || ad->r > QLORA_MAX_RANK || ad->r % 8) return QLORA_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(ad->alpha)) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(ad->A, 16) || !aligned(ad->B, 16)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

bool valid_dtype(qlora_dtype d) { return d == QLORA_F32 || d == QLORA_BF16; }

// T = X A^T for the tokens: writes s*T (bf16) to sT (if not null) and, if T_hi is
// not null, T as the bf16 pair (T_hi, T_lo) with T_hi + T_lo = T to ~16 bits.
// Rank-r GEMMs (T = X A^T, U = dY B): output tiles are few (M / 128), so when
// the caller's workspace holds the partial planes the K range is split over up
// to kMaxSplit CTAs per tile and the fp32 partials are summed, in split order,
// by splitk_finish_kernel.
constexpr int kMaxSplit = 8;
inline size_t split_part_bytes(int64_t M, int32_t r) {
  return align256(static_cast<size_t>(kMaxSplit) * static_cast<size_t>(M) * r * 4);
}
template <bool B_MN>
qlora_status launch_rank_gemm(const CUtensorMap &tmA, const CUtensorMap &tmB, GemmArgs g, float *part, int dev,
                              int sms, cudaStream_t st) {
  const int tiles = ((g.M_rows + 127) / 128) * ((g.N_cols + 63) / 64);
  int ks = part ? std::min(kMaxSplit, std::min(sms / std::max(1, tiles), g.k_steps / 4)) : 1;
  if (ks > 1) {
    g.k_per = (g.k_steps + ks - 1) / ks;
    ks = (g.k_steps + g.k_per - 1) / g.k_per;  // every split gets at least one step
  }
  if (ks <= 1) return launch_gemm<false, B_MN, false, 64, 1>(tmA, tmB, tmA, tmA, tmA, g, dev, sms, st);
  g.ksplit = ks;
  g.part = part;
  qlora_status s = launch_gemm<false, B_MN, false, 64, 1>(tmA, tmB, tmA, tmA, tmA, g, dev, sms, st);
  if (s != QLORA_OK) return s;
  const int64_t pairs = (int64_t)g.M_rows * g.N_cols / 2;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((pairs + 255) / 256, (int64_t)sms * 8));
  return launch_pdl(splitk_finish_kernel, dim3(grid), dim3(256), 0, st, g);
}

qlora_status run_lora_down(const void *X, const qlora_lora *ad, int64_t M, int64_t K, float s, void *sT,
                           void *T_hi, void *T_lo, float *part, uint32_t *status, int dev, int sms, cudaStream_t st,
                           float t_scale = 1.0f) {
  CUtensorMap tmX, tmA;
  if (!tmap_bf16(&tmX, X, K, M, 64, 128) || !tmap_bf16(&tmA, ad->A, K, ad->r, 64, 64)) return QLORA_ERR_CUDA;
  GemmArgs g{};
  g.M_rows = (int)M;
  g.N_cols = ad->r;
  g.k_steps = (int)(K / 64);
  g.out = sT;
  g.ldo = ad->r;
  g.out_f32 = 0;
  g.out_scale = s * t_scale;
  g.out_hi = static_cast<__nv_bfloat16 *>(T_hi);
  g.out_lo = static_cast<__nv_bfloat16 *>(T_lo);
  g.ld_hl = ad->r;
  g.hl_scale = t_scale;
  g.status = status;
  return launch_rank_gemm<false>(tmX, tmA, g, part, dev, sms, st);
}

// Least workspace the entry points accept (no K splitting of the rank-r GEMMs).
size_t min_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int for_backward) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0 || r > QLORA_MAX_RANK) return 0;
  const size_t mr = align256(static_cast<size_t>(M) * r * 2);  // one bf16 [M, r] buffer
  size_t bytes = QLORA_STATUS_BYTES;
  if (!for_backward) {
    // s*T: [M, r] bf16, or for the one-kernel decode path its tagged MMA
    // fragment entries (ceil(r/16) k-steps x two token halves x 32 lanes x 4
    // values x 8 bytes)
    const size_t frag = static_cast<size_t>((r + 15) / 16) * 2048;
    bytes += M <= kGemvMaxM ? std::max(mr, align256(frag)) : mr;
  } else {
    bytes += 4 * mr;                                // s*U (hi, lo), recomputed T (hi, lo)
  }
  return bytes;
}
// Float32 [M, N] base product of the multi-adapter decode's split path, placed
// after the minimum workspace.
size_t multi_base_bytes(int64_t M, int64_t N) { return align256(static_cast<size_t>(M) * N * 4); }
// Partial planes for K splitting, placed after the minimum workspace when the
// caller passed room for them.
float *split_part(void *ws, size_t ws_bytes, int64_t M, int64_t N, int64_t K, int32_t r, int for_backward) {
  if (!for_backward && M <= kGemvMaxM) return nullptr;
  const size_t lo = min_workspace_bytes(M, N, K, r, for_backward);
  if (ws_bytes < lo + split_part_bytes(M, r)) return nullptr;
  return reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + lo);
}

// Forward on a checked workspace: the base product reads X, the adapter branch
// reads Xl (X, or its dropped-out copy) and scales T by t_scale; part is the
// nullable K-split scratch.
qlora_status fwd_impl(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, const void *Xl, float t_scale,
                      int64_t M, void *Y, qlora_dtype y_dtype, void *T_save, void *ws, float *part,
                      qlora_stream_t stream) {
  qlora_status s;
  const int64_t N = W->rows, K = W->cols;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float sc = ad->alpha / static_cast<float>(ad->r);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  void *sT = wsb + QLORA_STATUS_BYTES;
  const size_t mr = align256(static_cast<size_t>(M) * ad->r * 2);

  if (M <= kGemvMaxM && Xl == X && aligned(W->scale_codes, 16) && ad->r % 8 == 0 && aligned(X, 16) &&
      aligned(ad->A, 16) && aligned(ad->B, 16)) {
    // one kernel per call: T, the fused dequant GEMV and the LoRA term
    const DecodePlan p = decode_plan(N, K, static_cast<int>(M), ad->r, sms, decode_smem_base(dev));
    CUtensorMap tmc, tmb;
    if (p.ok &&
        tmap_codes_gemv(&tmc, W->codes, N, K, static_cast<uint32_t>(p.WPR), static_cast<uint32_t>(16 * p.RPS)) &&
        tmap_brows(&tmb, ad->B, N, ad->r, static_cast<uint32_t>(16 * p.RPS))) {
      DecodeArgs g{};
      g.codes = W->codes;
      g.scale_codes = W->scale_codes;
      g.c2 = W->c2;
      g.scale_format = W->scale_format;
      g.X = static_cast<const __nv_bfloat16 *>(X);
      g.A = static_cast<const __nv_bfloat16 *>(ad->A);
      g.B = static_cast<const __nv_bfloat16 *>(ad->B);
      g.N = N;
      g.K = K;
      g.M = static_cast<int>(M);
      g.r = ad->r;
      g.s = sc;
      g.Y = Y;
      g.y_f32 = y_dtype == QLORA_F32;
      g.stf_g = reinterpret_cast<uint64_t *>(sT);
      __nv_bfloat16 *th = static_cast<__nv_bfloat16 *>(T_save);
      g.T_hi = th;
      g.T_lo = th ? th + M * ad->r : nullptr;
      g.status = status_ptr(ws);
      g.bar_count = status_ptr(ws) + 1;
      g.bar_gen = status_ptr(ws) + 2;
      g.G = p.G;
      g.units = p.units;
      g.units_max = p.units_max;
      g.WPR = p.WPR;
      g.RPS = p.RPS;
      g.stages = p.stages;
      g.F = p.F;
      g.stf_bytes = p.stf_bytes;
      g.brow_unit_bytes = p.brow_unit_bytes;
      g.lay = p.lay;
      g.lay_base = p.base;
      return launch_decode(p, g, tmc, tmb, dev, st);
    }
  }
  if (M <= kGemvMaxM) {
    __nv_bfloat16 *th = static_cast<__nv_bfloat16 *>(T_save);
    auto down = M > 8 ? lora_down_small_kernel<2> : lora_down_small_kernel<1>;
    down<<<(ad->r + 15) / 16, kLoraDownThreads, 0, st>>>(static_cast<const __nv_bfloat16 *>(Xl),
                                                        static_cast<const __nv_bfloat16 *>(ad->A), (int)M, K, ad->r, sc,
                                                        static_cast<__nv_bfloat16 *>(sT), th,
                                                        th ? th + M * ad->r : nullptr, t_scale);
    if ((s = launch_status()) != QLORA_OK) return s;
    GemvArgs g{};
    g.codes = W->codes; g.scale_codes = W->scale_codes; g.c2 = W->c2; g.scale_format = W->scale_format;
    g.N = N; g.K = K; g.M = (int)M;
    g.X = static_cast<const __nv_bfloat16 *>(X);
    g.sT = static_cast<const __nv_bfloat16 *>(sT);
    g.B = static_cast<const __nv_bfloat16 *>(ad->B);
    g.r = ad->r;
    g.Y = Y; g.y_f32 = y_dtype == QLORA_F32;
    g.partial = reinterpret_cast<float *>(wsb + QLORA_STATUS_BYTES + mr);
    g.status = status_ptr(ws);
    CUtensorMap tmc;
    const bool staged = gemv_bulk_ok(N, K) &&
                        tmap_codes_gemv(&tmc, W->codes, N, K, static_cast<uint32_t>((K < 4096 ? K : 4096) / 256));
    return launch_gemv(g, staged ? &tmc : nullptr, dev, sms, st);
  }

  {
    __nv_bfloat16 *th = static_cast<__nv_bfloat16 *>(T_save);
    if ((s = run_lora_down(Xl, ad, M, K, sc, sT, th, th ? th + M * ad->r : nullptr, part, status_ptr(ws), dev, sms,
                           st, t_scale)) != QLORA_OK)
      return s;
  }

  CUtensorMap tmX, tmCodes, tmT, tmCodesPair;
  if (!tmap_bf16(&tmX, X, K, M, 64, 128) || !tmap_bf16(&tmT, sT, ad->r, M, 64, 128) ||
      !make_tmap(&tmCodes, W->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 32, 256, false) ||
      !make_tmap(&tmCodesPair, W->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 32, 128, false))
    return QLORA_ERR_CUDA;
  GemmArgs g{};
  g.M_rows = (int)M;
  g.N_cols = (int)N;
  g.k_steps = (int)(K / 64);
  g.lora_steps = (ad->r + 63) / 64;
  g.lora_r = ad->r;
  g.out = Y;
  g.ldo = N;
  g.out_f32 = y_dtype == QLORA_F32;
  g.out_scale = 1.0f;
  g.scale_codes = W->scale_codes;
  g.c2 = W->c2;
  g.scale_format = W->scale_format;
  g.w_rows = N;
  g.w_cols = K;
  g.lora_b2 = static_cast<const __nv_bfloat16 *>(ad->B);
  g.lora_ld = ad->r;
  g.status = status_ptr(ws);
  if (M >= kPairMinRows) {
    s = launch_gemm_pair<false, kFusedMT>(tmX, tmT, tmCodesPair, g, dev, st);
    if (s != QLORA_ERR_UNSUPPORTED_SHAPE) return s;
  }
  return launch_gemm<false, false, true, 256, kFusedMT>(tmX, tmX, tmT, tmX, tmCodes, g, dev, sms, st);
}

// Backward on a checked workspace: dA and a recomputed T read Xl (X, or its
// dropped-out copy) with t_scale; keep (nullable) masks the adapter term of dX.
qlora_status bwd_impl(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, const void *Xl, float t_scale,
                      const void *keep, const void *dY, int64_t M, const void *T_saved, void *dX, qlora_dtype dx_dtype,
                      void *dA, void *dB, qlora_dtype grad_dtype, void *ws, float *part, qlora_stream_t stream) {
  qlora_status s;
  const int64_t N = W->rows, K = W->cols;
  (void)X;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float sc = ad->alpha / static_cast<float>(ad->r);
  const int r = ad->r;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  const size_t mr = align256(static_cast<size_t>(M) * r * 2);
  void *sU_hi = wsb + QLORA_STATUS_BYTES;
  void *sU_lo = wsb + QLORA_STATUS_BYTES + mr;
  uint32_t *status = status_ptr(ws);

  const void *T_hi = T_saved;
  const void *T_lo = T_saved ? static_cast<const __nv_bfloat16 *>(T_saved) + M * r : nullptr;
  if (!T_saved) {
    void *th = wsb + QLORA_STATUS_BYTES + 2 * mr, *tl = wsb + QLORA_STATUS_BYTES + 3 * mr;
    if ((s = run_lora_down(Xl, ad, M, K, sc, nullptr, th, tl, part, status, dev, sms, st, t_scale)) != QLORA_OK)
      return s;
    T_hi = th;
    T_lo = tl;
  }
  // U = dY B, kept as the bf16 pair (hi, lo) of s*U
  {
    CUtensorMap tmDY, tmB;
    if (!tmap_bf16(&tmDY, dY, N, M, 64, 128) || !tmap_bf16(&tmB, ad->B, r, N, 64, 64)) return QLORA_ERR_CUDA;
    GemmArgs g{};
    g.M_rows = (int)M;
    g.N_cols = r;
    g.k_steps = (int)((N + 63) / 64);
    g.out_hi = static_cast<__nv_bfloat16 *>(sU_hi);
    g.out_lo = static_cast<__nv_bfloat16 *>(sU_lo);
    g.ld_hl = r;
    g.hl_scale = sc;
    g.status = status;
    if ((s = launch_rank_gemm<true>(tmDY, tmB, g, part, dev, sms, st)) != QLORA_OK) return s;
  }
  // dX = dY W' + (s U) A
  {
    CUtensorMap tmDY, tmU, tmCodes, tmCodesPair;
    if (!tmap_bf16(&tmDY, dY, N, M, 64, 128) || !tmap_bf16(&tmU, sU_hi, r, M, 64, 128) ||
        !make_tmap(&tmCodes, W->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 128, 64, false) ||
        !make_tmap(&tmCodesPair, W->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 64, 64, false))
      return QLORA_ERR_CUDA;
    GemmArgs g{};
    g.M_rows = (int)M;
    g.N_cols = (int)K;
    g.k_steps = (int)((N + 63) / 64);
    g.lora_steps = keep ? 0 : (r + 63) / 64;  // with dropout the adapter term is added masked, below
    g.lora_r = r;
    g.out = dX;
    g.ldo = K;
    g.out_f32 = dx_dtype == QLORA_F32;
    g.out_scale = 1.0f;
    g.scale_codes = W->scale_codes;
    g.c2 = W->c2;
    g.scale_format = W->scale_format;
    g.w_rows = N;
    g.w_cols = K;
    g.lora_b2 = static_cast<const __nv_bfloat16 *>(ad->A);
    g.lora_ld = K;
    g.status = status;
    s = M >= kPairMinRows ? launch_gemm_pair<true, kFusedMT>(tmDY, tmU, tmCodesPair, g, dev, st)
                          : QLORA_ERR_UNSUPPORTED_SHAPE;
    if (s == QLORA_ERR_UNSUPPORTED_SHAPE)
      s = launch_gemm<false, true, true, 256, kFusedMT>(tmDY, tmDY, tmU, tmDY, tmCodes, g, dev, sms, st);
    if (s != QLORA_OK) return s;
  }
  // dropout: dX += keep * ((s U) A) / (1 - p)
  if (keep) {
    CUtensorMap tmU, tmAl;
    if (!tmap_bf16(&tmU, sU_hi, r, M, 64, 128) || !tmap_bf16(&tmAl, ad->A, K, r, 64, 64)) return QLORA_ERR_CUDA;
    GemmArgs g{};
    g.M_rows = (int)M;
    g.N_cols = (int)K;
    g.k_steps = (r + 63) / 64;
    g.out = dX;
    g.ldo = K;
    g.out_f32 = dx_dtype == QLORA_F32;
    g.out_scale = 1.0f;
    g.keep = static_cast<const uint8_t *>(keep);
    g.keep_scale = t_scale;
    g.status = status;
    if ((s = launch_gemm<false, true, false, 128, 1>(tmU, tmAl, tmU, tmU, tmU, g, dev, sms, st)) != QLORA_OK)
      return s;
  }
  // dA^T [K, r] = X^T (s U_hi + s U_lo)  -> stored transposed into dA [r, K], and
  // dB [N, r] = s dY^T (T_hi + T_lo): independent, one launch for both
  {
    CUtensorMap tmXt, tmUh, tmUl, tmDYt, tmTh, tmTl;
    if (!tmap_bf16(&tmXt, Xl, K, M, 64, 64) || !tmap_bf16(&tmUh, sU_hi, r, M, 64, 64) ||
        !tmap_bf16(&tmUl, sU_lo, r, M, 64, 64) || !tmap_bf16(&tmDYt, dY, N, M, 64, 64) ||
        !tmap_bf16(&tmTh, T_hi, r, M, 64, 64) || !tmap_bf16(&tmTl, T_lo, r, M, 64, 64))
      return QLORA_ERR_CUDA;
    GemmArgs ga{};
    ga.M_rows = (int)K;
    ga.N_cols = r;
    ga.k_steps = (int)((M + 63) / 64);
    ga.hilo_cols = 1;
    ga.out = dA;
    ga.ldo = K;
    ga.out_f32 = grad_dtype == QLORA_F32;
    ga.out_transpose = 1;
    ga.out_scale = t_scale;
    ga.status = status;
    GemmArgs gb{};
    gb.M_rows = (int)N;
    gb.N_cols = r;
    gb.k_steps = (int)((M + 63) / 64);
    gb.hilo_cols = 1;
    gb.out = dB;
    gb.ldo = r;
    gb.out_f32 = grad_dtype == QLORA_F32;
    gb.out_scale = sc;
    gb.status = status;
    if ((s = launch_gemm<true, true, false, 128, 1>(tmXt, tmUh, tmXt, tmUl, tmXt, ga, dev, sms, st, &gb, &tmDYt,
                                                     &tmTh, &tmTl)) != QLORA_OK)
      return s;
  }
  return QLORA_OK;
}


}  // namespace

extern "C" {

int qlora_abi_version(void) { return QLORA_NF4_ABI_VERSION; }

void qlora_nf4_codebook(float out[16]) {
  if (!out) return;
  const float *lv = nf4_levels_host();
  for (int i = 0; i < 16; ++i) out[i] = lv[i];
}

size_t qlora_nf4_storage_bytes(int64_t rows, int64_t cols, size_t *codes_bytes, size_t *scale_codes_bytes,
                               size_t *c2_bytes) {
  if (rows <= 0 || cols <= 0 || cols % QLORA_BLOCK) return 0;
  const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(cols);
  const size_t nb = n / QLORA_BLOCK;
  const size_t ng = (nb + QLORA_GROUP - 1) / QLORA_GROUP;
  if (codes_bytes) *codes_bytes = n / 2;
  if (scale_codes_bytes) *scale_codes_bytes = nb;
  if (c2_bytes) *c2_bytes = ng * sizeof(float);
  return n / 2 + nb + ng * sizeof(float);
}

size_t qlora_workspace_bytes_multi(int64_t M, int64_t N, int64_t K, int32_t r) {
  const size_t lo = min_workspace_bytes(M, N, K, r, 0);
  if (lo == 0 || M > kGemvMaxM) return 0;
  return lo + multi_base_bytes(M, N);
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int for_backward) {
  const size_t lo = min_workspace_bytes(M, N, K, r, for_backward);
  if (lo == 0) return 0;
  if (!for_backward && M <= kGemvMaxM) return lo;
  return lo + split_part_bytes(M, r);
}

qlora_status qlora_nf4_quantize(const void *W, qlora_dtype w_dtype, const qlora_nf4_tensor *out, void *ws,
                                qlora_stream_t stream) {
  qlora_status s = check_nf4(out);
  if (s != QLORA_OK) return s;
  if (!W || !ws) return QLORA_ERR_INVALID_ARGUMENT;
  if (!valid_dtype(w_dtype)) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(W, 16) || !aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  const HostCellTable &ht = cell_table();
  if (!ht.ok) return QLORA_ERR_CUDA;
  CodeCellTable t;
  std::memcpy(t.thr, ht.thr, sizeof(t.thr));
  std::memcpy(t.base, ht.base, sizeof(t.base));
  const int64_t nb = out->rows * out->cols / QLORA_BLOCK;
  const int64_t ng = (nb + QLORA_GROUP - 1) / QLORA_GROUP;
  if (ng > 0x7fffffff) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (w_dtype == QLORA_BF16)
    nf4_quantize_kernel<__nv_bfloat16><<<(unsigned)ng, kQuantThreads, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(W), nb, out->codes, out->scale_codes, out->c2, status_ptr(ws), t,
        out->scale_format);
  else
    nf4_quantize_kernel<float><<<(unsigned)ng, kQuantThreads, 0, st>>>(
        static_cast<const float *>(W), nb, out->codes, out->scale_codes, out->c2, status_ptr(ws), t,
        out->scale_format);
  return launch_status();
}

qlora_status qlora_nf4_dequantize(const qlora_nf4_tensor *w, void *W_out, qlora_dtype out_dtype,
                                  qlora_stream_t stream) {
  qlora_status s = check_nf4(w);
  if (s != QLORA_OK) return s;
  if (!W_out || !valid_dtype(out_dtype)) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(W_out, 16)) return QLORA_ERR_MISALIGNED;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  const int64_t nchunks = w->rows * w->cols / 32;
  const int64_t want = (nchunks + kDequantThreads - 1) / kDequantThreads;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 16));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (out_dtype == QLORA_BF16) {
    // one warp step per 1024 weights; enough CTAs for about two steps per warp
    const int64_t nweights = w->rows * w->cols;
    const int64_t wsteps = (nweights + 1023) / 1024;
    const int64_t ctas = (wsteps + 2 * kDequantWarps - 1) / (2 * kDequantWarps);
    const unsigned gb = (unsigned)std::max<int64_t>(1, std::min<int64_t>(ctas, (int64_t)1 << 20));
    if (reinterpret_cast<uintptr_t>(W_out) % 32 == 0)
      nf4_dequantize_bf16_v8_kernel<<<gb, kDequantThreads, 0, st>>>(w->codes, w->scale_codes, w->c2, nweights,
                                                                   static_cast<__nv_bfloat16 *>(W_out), w->scale_format);
    else
      nf4_dequantize_bf16_kernel<<<gb, kDequantThreads, 0, st>>>(w->codes, w->scale_codes, w->c2, nweights,
                                                                 static_cast<__nv_bfloat16 *>(W_out), w->scale_format);
  } else
    nf4_dequantize_kernel<float><<<grid, kDequantThreads, 0, st>>>(w->codes, w->scale_codes, w->c2, nchunks,
                                                                   static_cast<float *>(W_out), w->scale_format);
  return launch_status();
}

qlora_status qlora_linear_fwd(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, int64_t M, void *Y,
                              qlora_dtype y_dtype, void *T_save, void *ws, size_t ws_bytes,
                              qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(ad)) != QLORA_OK) return s;
  if (!X || !Y || !ws || M < 1 || M > (int64_t(1) << 30) || !valid_dtype(y_dtype)) return QLORA_ERR_INVALID_ARGUMENT;
  if (W->rows % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256) || (T_save && !aligned(T_save, 16)))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  if (ws_bytes < min_workspace_bytes(M, N, K, ad->r, 0)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  return fwd_impl(W, ad, X, X, 1.0f, M, Y, y_dtype, T_save, ws, split_part(ws, ws_bytes, M, N, K, ad->r, 0),
                  stream);
}

qlora_status qlora_linear_bwd(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, const void *dY,
                              int64_t M, const void *T_saved, void *dX, qlora_dtype dx_dtype, void *dA, void *dB,
                              qlora_dtype grad_dtype, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(ad)) != QLORA_OK) return s;
  if (!X || !dY || !dX || !dA || !dB || !ws || M < 1 || M > (int64_t(1) << 30)) return QLORA_ERR_INVALID_ARGUMENT;
  if (!valid_dtype(dx_dtype) || !valid_dtype(grad_dtype)) return QLORA_ERR_INVALID_ARGUMENT;
  if (W->rows % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(dY, 16) || !aligned(dX, 16) || !aligned(dA, 16) || !aligned(dB, 16) ||
      !aligned(ws, 256) || (T_saved && !aligned(T_saved, 16)))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  if (ws_bytes < min_workspace_bytes(M, N, K, ad->r, 1)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  return bwd_impl(W, ad, X, X, 1.0f, nullptr, dY, M, T_saved, dX, dx_dtype, dA, dB, grad_dtype, ws,
                  split_part(ws, ws_bytes, M, N, K, ad->r, 1), stream);
}

size_t qlora_workspace_bytes_dropout(int64_t M, int64_t N, int64_t K, int32_t r, int for_backward) {
  const size_t lo = min_workspace_bytes(M, N, K, r, for_backward);
  if (lo == 0) return 0;
  const size_t xm = align256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
  if (!for_backward && M <= kGemvMaxM) return lo + xm;
  return lo + xm + split_part_bytes(M, r);
}

namespace {
// X * keep into the workspace right after its minimum part; returns the copy and
// the K-split scratch after it (null when the workspace has no room for it).
qlora_status dropout_input(const void *X, const void *keep, int64_t M, int64_t N, int64_t K, int32_t r,
                           int for_backward, void *ws, size_t ws_bytes, int sms, cudaStream_t st, void **Xm,
                           float **part) {
  const size_t lo = min_workspace_bytes(M, N, K, r, for_backward);
  const size_t xm = align256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
  if (ws_bytes < lo + xm) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  *Xm = wsb + lo;
  *part = (for_backward || M > kGemvMaxM) && ws_bytes >= lo + xm + split_part_bytes(M, r)
              ? reinterpret_cast<float *>(wsb + lo + xm)
              : nullptr;
  const int64_t n8 = M * K / 8;
  const unsigned grid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, (int64_t)sms * 8)));
  keep_mask_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(X), static_cast<const uint8_t *>(keep), n8,
                                         static_cast<__nv_bfloat16 *>(*Xm));
  return launch_status();
}
}  // namespace

qlora_status qlora_linear_fwd_dropout(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, const void *keep,
                                      float p, int64_t M, void *Y, qlora_dtype y_dtype, void *T_save, void *ws,
                                      size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(ad)) != QLORA_OK) return s;
  if (!X || !keep || !Y || !ws || M < 1 || M > (int64_t(1) << 30) || !valid_dtype(y_dtype) || !(p >= 0.0f && p < 1.0f))
    return QLORA_ERR_INVALID_ARGUMENT;
  if (W->rows % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(keep, 16) || !aligned(Y, 16) || !aligned(ws, 256) ||
      (T_save && !aligned(T_save, 16)))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  if (ws_bytes < min_workspace_bytes(M, N, K, ad->r, 0)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void *Xm;
  float *part;
  if ((s = dropout_input(X, keep, M, N, K, ad->r, 0, ws, ws_bytes, sms, st, &Xm, &part)) != QLORA_OK) return s;
  return fwd_impl(W, ad, X, Xm, 1.0f / (1.0f - p), M, Y, y_dtype, T_save, ws, part, stream);
}

qlora_status qlora_linear_bwd_dropout(const qlora_nf4_tensor *W, const qlora_lora *ad, const void *X, const void *dY,
                                      const void *keep, float p, int64_t M, const void *T_saved, void *dX,
                                      qlora_dtype dx_dtype, void *dA, void *dB, qlora_dtype grad_dtype, void *ws,
                                      size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(ad)) != QLORA_OK) return s;
  if (!X || !dY || !keep || !dX || !dA || !dB || !ws || M < 1 || M > (int64_t(1) << 30) || !(p >= 0.0f && p < 1.0f))
    return QLORA_ERR_INVALID_ARGUMENT;
  if (!valid_dtype(dx_dtype) || !valid_dtype(grad_dtype)) return QLORA_ERR_INVALID_ARGUMENT;
  if (W->rows % 8) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || !aligned(dY, 16) || !aligned(keep, 16) || !aligned(dX, 16) || !aligned(dA, 16) ||
      !aligned(dB, 16) || !aligned(ws, 256) || (T_saved && !aligned(T_saved, 16)))
    return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  if (ws_bytes < min_workspace_bytes(M, N, K, ad->r, 1)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void *Xm;
  float *part;
  if ((s = dropout_input(X, keep, M, N, K, ad->r, 1, ws, ws_bytes, sms, st, &Xm, &part)) != QLORA_OK) return s;
  return bwd_impl(W, ad, X, Xm, 1.0f / (1.0f - p), keep, dY, M, T_saved, dX, dx_dtype, dA, dB, grad_dtype, ws, part,
                  stream);
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4_tensor *W, const qlora_lora *adapters, int32_t n_adapters,
                                    const int32_t *adapter_of_token, const void *X, int64_t M, void *Y,
                                    qlora_dtype y_dtype, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if (!adapters || n_adapters < 1 || !adapter_of_token || !X || !Y || !ws || M < 1 || M > kGemvMaxM ||
      !valid_dtype(y_dtype))
    return QLORA_ERR_INVALID_ARGUMENT;
  const int r = adapters[0].r;
  for (int32_t i = 0; i < n_adapters; ++i) {
    if ((s = check_lora(&adapters[i])) != QLORA_OK) return s;
    if (adapters[i].r != r) return QLORA_ERR_INVALID_ARGUMENT;
  }
  for (int64_t t = 0; t < M; ++t)
    if (adapter_of_token[t] < 0 || adapter_of_token[t] >= n_adapters) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  const int64_t N = W->rows, K = W->cols;
  if (!gemv_bulk_ok(N, K)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < min_workspace_bytes(M, N, K, r, 0)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  GemvArgs g{};
  for (int64_t t = 0; t < M; ++t) {
    const qlora_lora &ad = adapters[adapter_of_token[t]];
    g.ml.A[t] = static_cast<const __nv_bfloat16 *>(ad.A);
    g.ml.B[t] = static_cast<const __nv_bfloat16 *>(ad.B);
    g.ml.s[t] = ad.alpha / static_cast<float>(r);
  }
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  __nv_bfloat16 *sT = reinterpret_cast<__nv_bfloat16 *>(wsb + QLORA_STATUS_BYTES);
  // With room for a float32 [M, N] base product after the minimum workspace and a
  // rank with a power-of-two number of 16-byte pieces per row, the LoRA term runs
  // as its own pass over all SMs after the GEMV (lora_up_multi_kernel).
  const size_t ws_lo = min_workspace_bytes(M, N, K, r, 0);
  const int P = r / 8;
  const bool split = (P & (P - 1)) == 0 && ws_bytes >= ws_lo + multi_base_bytes(M, N);
  float *Yb = split ? reinterpret_cast<float *>(wsb + ws_lo) : nullptr;
  // s T on the SMs the GEMV leaves free (at least eight CTAs, at most one warp per row)
  const int rows = static_cast<int>(M) * r, warps = kLoraDownMultiThreads / 32;
  int down = sms - gemv_grid_ctas(N, sms, true);
  if (down < 8) down = 8;
  if (down > (rows + warps - 1) / warps) down = (rows + warps - 1) / warps;
  lora_down_multi_kernel<<<down, kLoraDownMultiThreads, 0, st>>>(static_cast<const __nv_bfloat16 *>(X), g.ml,
                                                                   static_cast<int>(M), K, r, sT);
  if ((s = launch_status()) != QLORA_OK) return s;
  g.codes = W->codes; g.scale_codes = W->scale_codes; g.c2 = W->c2; g.scale_format = W->scale_format;
  g.N = N; g.K = K; g.M = (int)M;
  g.X = static_cast<const __nv_bfloat16 *>(X);
  g.sT = sT;
  g.B = g.ml.B[0];
  g.r = r;
  g.Y = split ? static_cast<void *>(Yb) : Y;
  g.y_f32 = split ? 1 : (y_dtype == QLORA_F32);
  g.status = status_ptr(ws);
  g.multi = split ? 2 : 1;
  CUtensorMap tmc;
  if (!tmap_codes_gemv(&tmc, W->codes, N, K, static_cast<uint32_t>((K < 4096 ? K : 4096) / 256)))
    return QLORA_ERR_CUDA;
  if ((s = launch_gemv(g, &tmc, dev, sms, st)) != QLORA_OK || !split) return s;
  const int64_t rows_per_cta = static_cast<int64_t>(kLoraUpThreads / 32) * (32 / P) * kLoraUpRounds;
  const dim3 grid(static_cast<unsigned>((N + rows_per_cta - 1) / rows_per_cta), static_cast<unsigned>(M));
  return launch_pdl(lora_up_multi_kernel, grid, dim3(kLoraUpThreads), 0, st, static_cast<const float *>(Yb), g.ml,
                    static_cast<const __nv_bfloat16 *>(sT), N, r, Y, y_dtype == QLORA_F32 ? 1 : 0);
}

qlora_status qlora_lora_merge(const qlora_nf4_tensor *W, const qlora_lora *adapter, void *W_out,
                              qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(adapter)) != QLORA_OK) return s;
  if (!W_out) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(W_out, 16)) return QLORA_ERR_MISALIGNED;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  uint32_t *status = nullptr;
  if ((s = library_status_addr(dev, &status)) != QLORA_OK) return s;
  static std::once_flag flags[64];
  static qlora_status results[64];
  if ((s = set_smem(nf4_lora_merge_kernel, static_cast<int>(kMergeSmemBytes), dev, flags, results)) != QLORA_OK)
    return s;
  const int64_t N = W->rows, K = W->cols;
  const int r = adapter->r;
  // codes [N][K/2 bytes], box 128 B x 128 rows; B [N, r], box 64 ranks x 128 rows;
  // A [r, K], box 64 columns x 64 ranks; W_out [N, K], box 64 columns x 32 rows
  CUtensorMap tmCodes, tmB, tmA, tmOut;
  if (!make_tmap(&tmCodes, W->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 128, 128, true) ||
      !tmap_bf16(&tmB, adapter->B, r, N, 64, 128) || !tmap_bf16(&tmA, adapter->A, K, r, 64, 64) ||
      !tmap_bf16(&tmOut, W_out, K, N, 64, 32))
    return QLORA_ERR_CUDA;
  const int64_t tiles = ((N + kMergeBM - 1) / kMergeBM) * ((K + kMergeBN - 1) / kMergeBN);
  if (tiles >= (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  MergeArgs ma;
  ma.scale_codes = W->scale_codes;
  ma.c2 = W->c2;
  ma.N = N;
  ma.K = K;
  ma.r = r;
  ma.s = adapter->alpha / static_cast<float>(r);
  ma.fmt = W->scale_format;
  ma.status = status;
  nf4_lora_merge_kernel<<<grid, kMergeThreads, kMergeSmemBytes, reinterpret_cast<cudaStream_t>(stream)>>>(
      tmCodes, tmB, tmA, tmOut, ma);
  return launch_status();
}

qlora_status qlora_adamw_step(float *param, void *param_bf16, const float *grad, float *exp_avg, float *exp_avg_sq,
                              int64_t n, const qlora_adamw_hparams *hp, int64_t step, qlora_stream_t stream) {
  if (!param || !grad || !exp_avg || !exp_avg_sq || !hp || n < 1 || step < 1) return QLORA_ERR_INVALID_ARGUMENT;
  if (!(hp->lr >= 0.0f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
      !(hp->eps > 0.0f) || !(hp->weight_decay >= 0.0f) || !std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay))
    return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(param, 16) || !aligned(grad, 16) || !aligned(exp_avg, 16) || !aligned(exp_avg_sq, 16) ||
      (param_bf16 && !aligned(param_bf16, 8)))
    return QLORA_ERR_MISALIGNED;
  int dev, sms;
  qlora_status s;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  AdamWConsts c;
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), static_cast<double>(step));
  c.lr = hp->lr;
  c.beta1 = hp->beta1;
  c.beta2 = hp->beta2;
  c.eps = hp->eps;
  c.decay_factor = static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay);
  c.step_size = static_cast<float>(hp->lr / bc1);
  c.sqrt_bc2 = static_cast<float>(std::sqrt(bc2));
  const int64_t want = (n / 4 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8)));
  adamw_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      param, static_cast<__nv_bfloat16 *>(param_bf16), grad, exp_avg, exp_avg_sq, n, c);
  return launch_status();
}

}  // extern "C"

// Scratch of qlora_linear_fwd_noalloc: one static device array per GPU that
// loads the library.  Host code must not pass `g_noalloc_scratch` itself to a
// kernel (on the host it only names the symbol); its device address is looked up
// once per device with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

// Status word of the calls that take no workspace (qlora_lora_merge): one static
// device word per GPU, looked up like the scratch array.
static __device__ uint32_t g_library_status;

namespace {
// Only a successful lookup is cached: a lookup that fails (for example one made
// during a stream capture) is retried by the next call on that device.
qlora_status noalloc_scratch(int dev, void **out) {
  static std::mutex mu;
  static void *addr[64];
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return QLORA_OK;
}
qlora_status library_status_addr(int dev, uint32_t **out) {
  static std::mutex mu;
  static uint32_t *addr[64];
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_library_status) != cudaSuccess || !p) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    addr[dev] = static_cast<uint32_t *>(p);
  }
  *out = addr[dev];
  return QLORA_OK;
}
}  // namespace

extern "C" {

qlora_status qlora_linear_fwd_noalloc(const qlora_nf4_tensor *W, const qlora_lora *adapter, const void *X,
                                      int64_t M, void *Y, qlora_dtype y_dtype, void *T_save,
                                      qlora_stream_t stream) {
  qlora_status s = check_nf4(W);
  if (s != QLORA_OK) return s;
  if ((s = check_lora(adapter)) != QLORA_OK) return s;
  if (M < 1) return QLORA_ERR_INVALID_ARGUMENT;
  const size_t need = min_workspace_bytes(M, W->rows, W->cols, adapter->r, 0);
  if (need == 0) return QLORA_ERR_INVALID_ARGUMENT;
  if (need > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_UNSUPPORTED_SHAPE;
  int dev, sms;
  if ((s = check_device(&dev, &sms)) != QLORA_OK) return s;
  void *scratch = nullptr;
  if ((s = noalloc_scratch(dev, &scratch)) != QLORA_OK) return s;
  return qlora_linear_fwd(W, adapter, X, M, Y, y_dtype, T_save, scratch, QLORA_NOALLOC_SCRATCH_BYTES, stream);
}

qlora_status qlora_selftest_bounded_wait(void *ws, uint32_t limit_us, qlora_stream_t stream) {
  if (!ws || limit_us < 1 || limit_us > 2000000u) return QLORA_ERR_INVALID_ARGUMENT;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  qlora_status s;
  if ((s = check_device(nullptr, nullptr)) != QLORA_OK) return s;
  // the copy in flight reads the workspace header itself (QLORA_STATUS_BYTES)
  static_assert(kSelftestCopyBytes <= QLORA_STATUS_BYTES, "the copy stays inside the header");
  bounded_wait_selftest_kernel<<<1, kSelftestThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t *>(ws), status_ptr(ws), static_cast<uint64_t>(limit_us) * 1000u);
  return launch_status();
}

qlora_status qlora_clear_status(void *ws, qlora_stream_t stream) {
  if (!ws) return QLORA_ERR_INVALID_ARGUMENT;
  // words 0 (status) and 1 (arrival count); word 2 (generation) is kept
  return cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

qlora_status qlora_read_status(const void *ws, qlora_stream_t stream) {
  if (!ws) return QLORA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
  for (int code = 1; code < 32; ++code)
    if (word & (1u << code)) return static_cast<qlora_status>(code);
  return QLORA_OK;
}

qlora_status qlora_read_library_status(qlora_stream_t stream) {
  int dev;
  qlora_status s;
  if ((s = check_device(&dev, nullptr)) != QLORA_OK) return s;
  uint32_t *word_d = nullptr;
  if ((s = library_status_addr(dev, &word_d)) != QLORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, word_d, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
  if (word && cudaMemset(word_d, 0, sizeof(word)) != cudaSuccess) return QLORA_ERR_CUDA;
  for (int code = 1; code < 32; ++code)
    if (word & (1u << code)) return static_cast<qlora_status>(code);
  return QLORA_OK;
}

const char *qlora_status_string(qlora_status status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QLORA_ERR_MISALIGNED: return "misaligned pointer";
    case QLORA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case QLORA_ERR_NONFINITE: return "non-finite weight";
    case QLORA_ERR_TIMEOUT: return "device wait timed out";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

}  // extern "C"
