// Decode-shaped forward (M <= 16 tokens) of the NF4 linear layer with LoRA, one
// kernel per call:  Y [M, N] = X W'^T + s (X A^T) B^T  ("QLoRA" (Ultralytics
// glossary), "How QLoRA works": the frozen NF4 weight is dequantised right before
// the matmul and the LoRA path is added).
//
// The call is bound by reading the packed codes from HBM (0.5 B per weight) and
// by the instructions and shared-memory traffic of decoding them.  Design:
//
// * One CTA of 16 warps per SM, at most one per SM.  CTA c owns a contiguous
//   range of "units"; a unit is 16*RPS weight rows over the whole K (K <= 4096,
//   K % 256 == 0): RPS = 16 / (K / 256) row groups of 16 rows share a unit when
//   K < 4096.  Warp w owns row-group slot w / WPR and the 256-column slice
//   w % WPR (WPR = K / 256), keeping that slice of X in registers as fp16 MMA
//   fragments for the whole call.
// * Each unit's codes arrive in a ring of S stages, S units ahead of the
//   decode, as one tensor copy (TMA, 128-byte swizzle, so the eight rows a warp
//   reads at once fall into different banks) per unit and CTA: one copy
//   instruction per unit rather than one per warp, since a copy instruction
//   holds its issuing warp while the copy engine's queue is full.  The warp
//   that finishes a stage last (a shared-memory counter) refills it; no thread
//   executes a GPU-scope fence while the weight stream is in flight (measured
//   to hold the issuing warp for microseconds).  The B rows of all
//   the CTA's units come in one tensor copy per unit; the block scales of all
//   its rows are decoded once, S' = fl32(E4M3(q) * c2), into a float table.
//   Codes, scales, constants and B rows are requested before the kernel waits
//   for the preceding kernel of the stream (programmatic dependent launch), so
//   one call's weight stream overlaps the previous call's tail.  Nothing the kernel reads before that wait may be
//   written by a preceding kernel that triggers its dependents early: no kernel
//   of this library that writes a weight or an adapter does.  X and everything
//   derived from it are read after the wait.
// * Each code byte (two codes) indexes a 256-entry table of fp16 level pairs,
//   one copy per lane in a 64 KB-aligned shared table (one byte permute builds
//   the address); the pair is one register of an m16n8k16 A fragment
//   (rows = weight rows, columns = tokens), X enters as fp16 after an exact
//   per-token power-of-two scaling, and each 64-block's fp32 partial is scaled
//   by S' = fl32(E4M3(q) * c2).  The result equals X (L S')^T with L rounded to
//   fp16 (relative 2^-12): it differs from X W'^T only by the bf16 rounding of
//   W' = bf16(L S').
// * The warps' fp32 partials of each unit land in shared-memory slots without a
//   barrier; every F units (F slots; usually all of a CTA's units) the CTA meets
//   once and sums each row's warp slices in a fixed order (deterministic).
// * T = X A^T: the CTAs launched last compute ranks G-1-c, 2G-1-c, ... over all K
//   with the X fragments they already hold (A row in fragment row 0) and sum the
//   warps' slices in a fixed order.  They publish s*T as 64-bit entries
//   (bf16 value, generation tag), each one single store, and the saved
//   (T_hi, T_lo) pair.  The tag is the call's generation: every CTA reads the
//   generation word of the workspace header after the wait and adds one to an
//   arrival count; the last arrival resets the count and advances the
//   generation for the next call.  At the end every CTA copies the entries,
//   checks their tags (copying again until they all carry this call's tag) and
//   adds the LoRA term s T B^T of each row group on tensor cores.
//
// The workspace header (the first 256 bytes of ws) holds the status word, the
// arrival count and the generation; the count must be zero before a call (a
// zeroed workspace, or qlora_clear_status), and every completed call leaves it
// zero.  Every wait is bounded.
#pragma once

#include <mutex>

#include "gemv_kernel.cuh"
#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

constexpr int kDecWarps = 16;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMaxStages = 4;
constexpr uint32_t kDecLutBytes = 256 * 256;
constexpr uint32_t kDecSmemLimit = 232448;  // opt-in dynamic shared memory per CTA
constexpr uint32_t kDecWarpStage = 16 * 128;  // one warp's codes of one unit
constexpr uint32_t kDecStage = kDecWarps * kDecWarpStage;  // stage stride (a unit holds at most 16 slices)
constexpr int kDecScaleWords = 4 * kDecThreads;  // 4-block scale words decoded per prologue round
constexpr uint32_t kDecBarBytes = (kDecMaxStages + 2) * 8;

// Shared-memory placement (absolute shared addresses), computed on the host.
struct DecodeLayout {
  uint32_t lut;    // 64 KB-aligned pair table: entry v of lane l at v * 256 + l * 4
  uint32_t ring;   // codes, [stage][128-byte chunk kw][row of the unit][128 B] swizzled, 1024-aligned
  uint32_t sf;     // decoded block scales S', [row of the CTA][decode_sf_stride(K/64)] floats
  uint32_t brows;  // the CTA's B rows, [unit][64-rank chunk][row of the unit][128 B] swizzled
  uint32_t red;    // partial sums, [F units][warp (stride 17 TR)][16 rows][TR]
  uint32_t yacc;   // reduced sums, [unit][row][TR]
  uint32_t stf;    // s*T entries, [r/16][NG][lane][4] u64 (bf16 value, tag)
  uint32_t bar;    // mbarriers: full[stage], then bbar (B rows), tbar (entries)
  uint32_t misc;   // u32: generation, abort flag, stage counters[kDecMaxStages]
  uint32_t end;
};

struct DecodeArgs {
  const uint8_t *codes;
  const uint8_t *scale_codes;
  const float *c2;
  int scale_format;           // qlora_scale_format of scale_codes
  const __nv_bfloat16 *X;
  const __nv_bfloat16 *A;
  const __nv_bfloat16 *B;
  int64_t N, K;
  int M, r;
  float s;
  void *Y;
  int y_f32;
  uint64_t *stf_g;            // workspace: s*T entries (written and read by this kernel)
  uint32_t brow_unit_bytes;   // one unit's B rows (all chunks)
  __nv_bfloat16 *T_hi, *T_lo; // nullable
  uint32_t *status;           // workspace header word 0
  uint32_t *bar_count;        // workspace header word 1
  uint32_t *bar_gen;          // workspace header word 2
  int G;                      // grid size (<= SMs, one CTA per SM)
  int units, units_max;       // units in all, most units of one CTA
  int WPR, RPS;               // warps per row group (K / 256), row groups per unit
  int stages;                 // ring depth
  int F;                      // units per round (partial-sum slots)
  uint32_t stf_bytes;
  DecodeLayout lay;
  uint32_t lay_base;          // shared address the host assumed for the dynamic window
};

// Shapes the kernel takes: K a multiple of 256 up to 4096 (one unit spans all of
// K), and rank up to 64 or a multiple of 64 up to 256 (the B-row copy moves
// 64-rank chunks).
inline bool decode_shape_ok(int64_t K, int r) {
  return K >= 256 && K <= 4096 && K % 256 == 0 && r <= 256 && (r <= 64 || r % 64 == 0);
}

struct DecodePlan {
  int G = 0, units = 0, units_max = 0, WPR = 0, RPS = 0, stages = 0, F = 0, NG = 1, TR = 8, chunks = 1;
  uint32_t ring_bytes = 0, sf_bytes = 0, brows_bytes = 0, brow_unit_bytes = 0, stf_bytes = 0, red_unit_bytes = 0,
           yacc_bytes = 0;
  DecodeLayout lay{};
  uint32_t base = 0;
  int dyn_bytes = 0;
  bool ok = false;
};

inline uint32_t dec_align(uint32_t x, uint32_t a) { return (x + a - 1) & ~(a - 1); }

// Row stride (floats) of the decoded scale table for K/64 = nbk blocks per row:
// an odd multiple of 4 modulo 32, so the eight rows a warp reads at once (16
// bytes each) fall into different banks.
__host__ __device__ inline int decode_sf_stride(int nbk) { return nbk + (((nbk >> 2) & 1) ? 8 : 4); }

// s*T entries: ceil(r/16) k-steps x NG token halves x 32 lanes x 4 bf16 values,
// 8 bytes each.
inline uint32_t decode_stf_bytes(int r, int ng) { return static_cast<uint32_t>(((r + 15) / 16) * ng * 32 * 4 * 8); }

// Places the buffers around the 64 KB-aligned table for a dynamic window that
// starts at shared address `base`.
inline DecodeLayout decode_layout(uint32_t base, uint32_t ring_bytes, uint32_t sf_bytes, uint32_t brows_bytes,
                                  uint32_t red_bytes, uint32_t yacc_bytes, uint32_t stf_bytes) {
  DecodeLayout L{};
  L.lut = (base + 0xffffu) & ~0xffffu;
  uint32_t lo_next = base, hi_next = L.lut + kDecLutBytes;
  auto place = [&](uint32_t bytes, uint32_t align) -> uint32_t {
    const uint32_t lo = dec_align(lo_next, align);
    if (lo + bytes <= L.lut) {
      lo_next = lo + bytes;
      return lo;
    }
    const uint32_t hi = dec_align(hi_next, align);
    hi_next = hi + bytes;
    return hi;
  };
  L.ring = place(ring_bytes, 1024);
  L.brows = place(brows_bytes, 1024);
  L.red = place(red_bytes, 16);
  L.sf = place(sf_bytes, 16);
  L.yacc = place(yacc_bytes, 16);
  L.stf = place(stf_bytes, 16);
  L.bar = place(kDecBarBytes, 8);
  L.misc = place(32, 16);
  L.end = hi_next > lo_next ? hi_next : lo_next;
  return L;
}

// Work split and shared-memory plan for M tokens, W [N, K], rank r on `sms` SMs
// with the dynamic window at `base`.  Prefers three stages and as many
// partial-sum slots as the CTA has units; ok is false when two stages and one
// slot do not fit.
inline DecodePlan decode_plan(int64_t N, int64_t K, int M, int r, int sms, uint32_t base) {
  DecodePlan p;
  if (!decode_shape_ok(K, r) || M < 1 || M > kGemvMaxM || N < 1 || r < 1) return p;
  p.NG = M > 8 ? 2 : 1;
  p.TR = M > 8 ? 16 : 8;
  p.WPR = static_cast<int>(K / 256);
  p.RPS = kDecWarps / p.WPR;
  const int64_t rows_per_unit = 16LL * p.RPS;
  const int64_t units = (N + rows_per_unit - 1) / rows_per_unit;
  if (units > (int64_t(1) << 24)) return p;
  p.units = static_cast<int>(units);
  p.G = p.units < sms ? p.units : sms;
  p.units_max = (p.units + p.G - 1) / p.G;  // CTAs below units % G take one unit more
  const int64_t crows = p.units_max * rows_per_unit;
  p.chunks = (r + 63) / 64;
  p.sf_bytes = static_cast<uint32_t>(crows * decode_sf_stride(static_cast<int>(K / 64)) * 4);
  p.brow_unit_bytes = static_cast<uint32_t>(p.chunks * rows_per_unit * 128);
  p.brows_bytes = p.units_max * p.brow_unit_bytes;
  p.stf_bytes = decode_stf_bytes(r, p.NG);
  p.red_unit_bytes = static_cast<uint32_t>(kDecWarps * 17 * p.TR * 4);
  p.yacc_bytes = static_cast<uint32_t>(crows * p.TR * 4);
  if (crows * K / 64 > (int64_t(1) << 20)) return p;
  const int smax = p.units_max < 3 ? (p.units_max < 2 ? 2 : p.units_max) : 3;
  for (int st = smax; st >= 2; --st)
    for (int f = p.units_max; f >= 1; --f) {
      const uint32_t ring = static_cast<uint32_t>(st) * kDecStage;
      const DecodeLayout L =
          decode_layout(base, ring, p.sf_bytes, p.brows_bytes, f * p.red_unit_bytes, p.yacc_bytes, p.stf_bytes);
      if (L.end - base <= kDecSmemLimit) {
        p.lay = L;
        p.stages = st;
        p.F = f;
        p.ring_bytes = ring;
        p.base = base;
        p.dyn_bytes = static_cast<int>(L.end - base);
        p.ok = true;
        return p;
      }
    }
  return p;
}

// fp16 bit pattern of level j (a select chain over compile-time constants: no
// constant-memory fetch in the kernel's prologue).
__device__ __forceinline__ uint32_t nf4_level_f16_bits(int j) {
  return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(nf4_level(j))));
}

__device__ __forceinline__ uint4 ld_cg_u128(const void *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

template <int NG>
__global__ void __launch_bounds__(kDecThreads, 1)
    nf4_decode_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_b,
                      const DecodeArgs a, int dyn_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr int TR = NG == 1 ? 8 : 16;  // token columns of a partial-sum row
  constexpr int BG = 2;                 // blocks whose MMA chains run interleaved
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;

  const uint32_t base = ptx::smem_addr(smem_raw);
  const DecodeLayout &Lay = a.lay;
  if (base != a.lay_base || Lay.end > base + static_cast<uint32_t>(dyn_bytes) || a.stages < 2 ||
      a.stages > kDecMaxStages || a.F < 1) {
    if (tid == 0) raise_status(a.status, QLORA_ERR_CUDA);  // the host sized the window for another start
    return;
  }
  auto at = [&](uint32_t addr) { return smem_raw + (addr - base); };
  uint64_t *full = reinterpret_cast<uint64_t *>(at(Lay.bar));  // [stage][warp]
  uint64_t *bbar = full + kDecMaxStages, *tbar = bbar + 1;
  volatile uint32_t *flags = reinterpret_cast<volatile uint32_t *>(at(Lay.misc));  // [0] generation, [1] abort
  uint32_t *ecnt = reinterpret_cast<uint32_t *>(at(Lay.misc)) + 2;  // warps done with each stage, cumulative
  const volatile int *abort_flag = reinterpret_cast<const volatile int *>(flags + 1);
  float *sf = reinterpret_cast<float *>(at(Lay.sf));
  float *yacc = reinterpret_cast<float *>(at(Lay.yacc));
  float *red = reinterpret_cast<float *>(at(Lay.red));
  const uint64_t *stf_s = reinterpret_cast<const uint64_t *>(at(Lay.stf));

  const int S = a.stages, F = a.F;
  // The CTAs launched first (lowest index) take the extra units: the last ones
  // start when the previous call's last CTAs leave their SMs.
  const int per = a.units / a.G, extra = a.units % a.G;
  const int U0 = static_cast<int>(blockIdx.x) * per + min(static_cast<int>(blockIdx.x), extra);
  const int nu = per + (static_cast<int>(blockIdx.x) < extra ? 1 : 0);
  const int WPR = a.WPR, RPS = a.RPS;
  const int rows_per_unit = 16 * RPS;
  const int rg_slot = warp / WPR, kw = warp % WPR;
  const bool active = rg_slot < RPS;
  const int64_t nbk = a.K / 64;
  const int64_t crow0 = static_cast<int64_t>(U0) * rows_per_unit;  // first row of this CTA
  const int crows = static_cast<int>(min(static_cast<int64_t>(nu) * rows_per_unit, a.N - crow0));
  const int r16 = (a.r + 15) & ~15;
  const int jfirst = a.G - 1 - static_cast<int>(blockIdx.x);
  const bool rank_cta = jfirst < r16;
  const uint64_t policy = ptx::l2_evict_first_policy();

  // ---- unit i's codes into ring slot i % S: one tensor copy of rows_per_unit
  // rows x K/2 bytes, stored as [chunk kw][row][16-byte unit XOR (row % 8)];
  // rows past N read as zeros (their block scales count zero as well).  This
  // warp reads chunk kw, rows 16 rg_slot .. 16 rg_slot + 15.
  const uint32_t unit_bytes = static_cast<uint32_t>(rows_per_unit * WPR * 128);
  const int nact = WPR * RPS;  // warps that decode
  uint8_t *ring_w = at(Lay.ring) + (kw * rows_per_unit + 16 * rg_slot) * 128;
  auto load_unit = [&](int i) {  // by one thread
    const int slot = i % S;
    ptx::mbar_arrive_expect_tx(full + slot, unit_bytes);
    ptx::tma_load_3d_hint(at(Lay.ring) + slot * kDecStage, &tm_codes, full + slot, 0, (U0 + i) * rows_per_unit, 0,
                          policy);
  };

  // ---- prologue (weights only)
  if (tid == 0) {
    ptx::prefetch_tmap(&tm_codes);
    ptx::prefetch_tmap(&tm_b);
    for (int st = 0; st < S; ++st) ptx::mbar_init(full + st, 1);
    ptx::mbar_init(bbar, 1);
    ptx::mbar_init(tbar, 1);
    ptx::fence_mbar_init();
    for (int i = 0; i < S && i < nu; ++i) load_unit(i);
    flags[0] = 0;
    flags[1] = 0;
    for (int st = 0; st < kDecMaxStages; ++st) ecnt[st] = 0;
  }
  __syncthreads();  // the barriers are initialised for every issuing lane
  if (lane == 0) {
    // B rows of unit u (all 64-rank chunks, ranks past r read as zeros), by warp u % 16
    for (int u = warp; u < nu; u += kDecWarps)
      ptx::tma_load_3d(at(Lay.brows) + u * a.brow_unit_bytes, &tm_b, bbar, 0, (U0 + u) * rows_per_unit, 0);
  }
  if (tid == 0) ptx::mbar_arrive_expect_tx(bbar, static_cast<uint32_t>(nu) * a.brow_unit_bytes);
  // block scales of the CTA's rows (crows * K/64 contiguous bytes from a 64-byte
  // aligned start) as 4-block words, with the second-level constant of each
  // word's group: loaded now, decoded once X is requested (their latency hides
  // behind the pair table and the wait)
  const int nwords = static_cast<int>(crows * nbk / 4);
  const uint32_t *sw = reinterpret_cast<const uint32_t *>(a.scale_codes + crow0 * nbk);
  uint32_t qv[4];
  float cv[4];
  auto load_scales = [&](int w0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int w = w0 + k * kDecThreads + tid;
      qv[k] = w < nwords ? __ldg(sw + w) : 0u;
      cv[k] = w < nwords ? __ldg(a.c2 + ((crow0 * nbk + 4 * w) >> 8)) : 0.0f;
    }
  };
  const int sfs = decode_sf_stride(static_cast<int>(nbk));  // row stride of the scale table (floats)
  auto store_scales = [&](int w0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int w = w0 + k * kDecThreads + tid;
      if (w < nwords) {
        const int row = (4 * w) / static_cast<int>(nbk), col = 4 * w - row * static_cast<int>(nbk);
        const float2 f01 = scale_code_value2(qv[k], a.scale_format);
        const float2 f23 = scale_code_value2(qv[k] >> 16, a.scale_format);
        *reinterpret_cast<float4 *>(sf + row * sfs + col) =
            make_float4(__fmul_rn(f01.x, cv[k]), __fmul_rn(f01.y, cv[k]), __fmul_rn(f23.x, cv[k]),
                        __fmul_rn(f23.y, cv[k]));
      }
    }
  };
  load_scales(0);
  // pair table: row v, lane l holds fp16 (L[v & 15], L[v >> 4]) at v * 256 + l * 4
  {
    const int v = tid >> 1;
    const uint32_t e = nf4_level_f16_bits(v & 15) | (nf4_level_f16_bits(v >> 4) << 16);
    uint4 *dst = reinterpret_cast<uint4 *>(at(Lay.lut + v * 256 + (tid & 1) * 64));
    const uint4 e4 = make_uint4(e, e, e, e);
    dst[0] = e4;
    dst[1] = e4;
    dst[2] = e4;
    dst[3] = e4;
  }

  griddep_launch_dependents();
  const uint32_t zero = griddep_wait_token();  // the preceding kernel is complete from here on
  // the call's generation, read before this CTA's arrival (so before the count
  // can complete), and the arrival itself (relaxed, its result used at the end)
  // (an acquiring load: the arrival cannot be performed before it)
  uint32_t arrive_old = 0u;
  if (tid == 0) {
    flags[0] = ptx::ld_acquire_gpu(a.bar_gen + zero);
    arrive_old = ptx::atom_add_relaxed_gpu(a.bar_count, 1u);
  }

  // ---- ranks of this CTA: G - 1 - c, 2G - 1 - c, ... (the CTAs launched last,
  // which also have the fewest units, take them); rank rows past r, up to the
  // next multiple of 16, are published as zeros.
  uint4 araw[4][2];
  auto load_arow = [&](int j) {
    const bool live = j < a.r && warp < WPR && g == 0;
    const __nv_bfloat16 *Arow = a.A + static_cast<int64_t>(live ? j : 0) * a.K + 256 * kw + 16 * q;
#pragma unroll
    for (int jb = 0; jb < 4; ++jb) {
      araw[jb][0] = live ? __ldg(reinterpret_cast<const uint4 *>(Arow + 64 * jb)) : make_uint4(0, 0, 0, 0);
      araw[jb][1] = live ? __ldg(reinterpret_cast<const uint4 *>(Arow + 64 * jb + 8)) : make_uint4(0, 0, 0, 0);
    }
  };

  // ---- X slice [256 kw, 256 kw + 256) as fp16 fragments: token g + 8 ng, k = 64 j + 16 q + ...
  uint32_t xf[4][4][NG][2];
  float unscale[NG][2];
  {
    const __nv_bfloat16 *X = a.X + zero;
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) {
      const int t = g + 8 * ng;
      uint4 raw[4][2];
      uint32_t mx = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (t < a.M) {
          const __nv_bfloat16 *src = X + static_cast<int64_t>(t) * a.K + 256 * kw + 64 * j + 16 * q;
          v0 = ld_cg_u128(src);
          v1 = ld_cg_u128(src + 8);
        }
        raw[j][0] = v0;
        raw[j][1] = v1;
      }
      // the decoded block scales, while the first token half's X is in flight
      if (ng == 0) store_scales(0);
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
      // bf16 bits -> exponent E with max |x| in [2^(E-1), 2^E); scale max into [2^14, 2^15)
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
      // exponent of token (2q + i + 8 ng), the C fragment's columns, lives in lane (2q + i) * 4
      unscale[ng][0] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q) * 4));
      unscale[ng][1] = pow2f(__shfl_sync(0xffffffffu, e, (2 * q + 1) * 4));
    }
  }

  // further rounds of block scales (more than 2048 words: rare)
  for (int w0 = kDecScaleWords; w0 < nwords; w0 += kDecScaleWords) {
    load_scales(w0);
    store_scales(w0);
  }
  __syncthreads();  // flags[0] (the generation) and the scale table are visible
  const uint32_t gen_next = flags[0] + 1u;
  // entries carry a bijective mix of the generation, so that a zeroed or
  // otherwise stale workspace does not look like this call's entries
  const uint32_t tag = gen_next * 0x9E3779B1u + 0x7F4A7C15u;

  // ---- T = X A^T for this CTA's ranks, published as (value, tag) entries
  if (rank_cta) {
    float *rred = red;  // [warp][16 tokens], before the first unit uses the slots
    for (int j = jfirst; j < r16; j += a.G) {
      const bool real = j < a.r;
      load_arow(j);
      if (real && warp < WPR) {
        uint32_t mx = 0;
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          const uint4 v0 = araw[jb][0], v1 = araw[jb][1];
          mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v0.x & 0x7fff7fffu, v0.y & 0x7fff7fffu),
                                     __vmaxu2(v0.z & 0x7fff7fffu, v0.w & 0x7fff7fffu)));
          mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v1.x & 0x7fff7fffu, v1.y & 0x7fff7fffu),
                                     __vmaxu2(v1.z & 0x7fff7fffu, v1.w & 0x7fff7fffu)));
        }
        uint32_t m16 = max(mx & 0xffffu, mx >> 16);
        m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
        m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 2));
        const int E = m16 ? static_cast<int>((m16 >> 7) & 0xff) - 126 : 15;
        const int ea = max(-100, min(100, E - 15));
        const float inva = pow2f(-ea);
        float acc[NG][4];
#pragma unroll
        for (int ng = 0; ng < NG; ++ng) acc[ng][0] = acc[ng][1] = acc[ng][2] = acc[ng][3] = 0.0f;
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint4 &v = araw[jb][s >> 1];
            const uint32_t a0 = bf16x2_to_f16x2_scaled((s & 1) ? v.z : v.x, inva);
            const uint32_t a2 = bf16x2_to_f16x2_scaled((s & 1) ? v.w : v.y, inva);
#pragma unroll
            for (int ng = 0; ng < NG; ++ng)
              mma_16816_f16_nv(acc[ng], a0, 0u, a2, 0u, xf[jb][s][ng][0], xf[jb][s][ng][1]);
          }
        }
        // row 0 of D: tokens 2q, 2q + 1 (+ 8 ng) in the lanes with g == 0
        if (g == 0) {
          const float ua = pow2f(ea);
#pragma unroll
          for (int ng = 0; ng < NG; ++ng) {
            rred[warp * 16 + 2 * q + 8 * ng] = acc[ng][0] * unscale[ng][0] * ua;
            rred[warp * 16 + 2 * q + 1 + 8 * ng] = acc[ng][1] * unscale[ng][1] * ua;
          }
        }
      }
      __syncthreads();
      if (warp == 0 && lane < a.M) {
        const int t = lane;
        float T = 0.0f;
        if (real)
          for (int w = 0; w < WPR; ++w) T += rred[w * 16 + t];
        // entry of rank j and token t: k-step j / 16, column kappa = j % 16 of the
        // B fragment: register kappa / 8, half kappa % 2, lane 4 (t % 8) + (kappa % 8) / 2
        const int kk = j >> 4, kap = j & 15;
        const int ln = 4 * (t & 7) + ((kap & 7) >> 1), ng = t >> 3;
        const uint64_t v = static_cast<uint64_t>(__bfloat16_as_ushort(__float2bfloat16_rn(T * a.s))) |
                           (static_cast<uint64_t>(tag) << 32);
        ptx::st_relaxed_gpu_u64(a.stf_g + (((kk * NG + ng) * 32 + ln) * 4 + (kap >> 3) * 2 + (kap & 1)), v);
        if (real && a.T_hi) {
          const __nv_bfloat16 h = __float2bfloat16_rn(T);
          a.T_hi[static_cast<int64_t>(t) * a.r + j] = h;
          a.T_lo[static_cast<int64_t>(t) * a.r + j] = __float2bfloat16_rn(T - __bfloat162float(h));
        }
      }
      __syncthreads();
    }
  }
  // Entries of tokens t >= M are never written or checked: they only feed output
  // columns of those tokens, which are discarded.


  // ---- main loop over this CTA's units.  Everything that changes from unit to
  // unit advances by a constant step (no division, no 64-bit arithmetic).
  const uint32_t laneword = (Lay.lut & 0xffff0000u) | static_cast<uint32_t>(lane * 4);
  // this thread's 8 code bytes of block j in its warp's slice: row g (+ 8 rows =
  // + 1024 bytes), 16-byte unit (2 j + q / 2) XOR g, bytes 8 (q % 2) onwards
  const uint32_t code_off = static_cast<uint32_t>(g * 128 + 8 * (q & 1));
  uint32_t code_xo[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) code_xo[j] = static_cast<uint32_t>(((2 * j + (q >> 1)) ^ g) << 4);
  // scales S' of blocks 4kw .. 4kw+3 of row g of this warp's row group in unit i
  const float *sfp = sf + (16 * rg_slot + g) * sfs + 4 * kw;
  const int unit_sf = rows_per_unit * sfs;
  // rows from row g of this warp's row group in unit i up to N
  const int64_t rows_left64 = a.N - (crow0 + 16 * rg_slot + g);
  int rows_left = static_cast<int>(rows_left64 < (int64_t(1) << 30) ? rows_left64 : (int64_t(1) << 30));
  int slot = 0, fs = 0, ring_round = 0;
  uint32_t phase = 0;
  for (int i = 0; i < nu; ++i) {
    float part[NG][4];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) part[ng][0] = part[ng][1] = part[ng][2] = part[ng][3] = 0.0f;
    // unit i's codes have landed in this warp's slot (every lane polls; the warp
    // decides together, and one that gave up leaves the decode to the status)
    const bool landed =
        !active || __all_sync(0xffffffffu, ptx::mbar_wait_spin(full + slot, phase, abort_flag));
    if (!landed && lane == 0) {  // the other warps leave their waits too
      raise_status(a.status, QLORA_ERR_TIMEOUT);
      flags[1] = 1;
    }
    if (active && landed) {
      const uint8_t *st = ring_w + slot * kDecStage;
      // block scales S' of blocks 4kw .. 4kw+3, rows g (h = 0) and g + 8 (h = 1)
      // of this warp's row group; rows past N count zero
      float S4[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 v = rows_left > 8 * h ? *reinterpret_cast<const float4 *>(sfp + 8 * h * sfs)
                                           : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        S4[h][0] = v.x;
        S4[h][1] = v.y;
        S4[h][2] = v.z;
        S4[h][3] = v.w;
      }
      const uint8_t *cb = st + code_off;
#pragma unroll
      for (int jg = 0; jg < 4; jg += BG) {
        uint2 cw[BG][2];
#pragma unroll
        for (int b = 0; b < BG; ++b) {
          cw[b][0] = *reinterpret_cast<const uint2 *>(cb + code_xo[jg + b]);
          cw[b][1] = *reinterpret_cast<const uint2 *>(cb + 1024 + code_xo[jg + b]);
        }
        float acc[BG][NG][4];
#pragma unroll
        for (int b = 0; b < BG; ++b)
#pragma unroll
          for (int ng = 0; ng < NG; ++ng) acc[b][ng][0] = acc[b][ng][1] = acc[b][ng][2] = acc[b][ng][3] = 0.0f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t p0 = (2 * s) & 3, p1 = (2 * s + 1) & 3;
          uint32_t af[BG][4];
#pragma unroll
          for (int b = 0; b < BG; ++b) {
            const uint32_t w0 = (s < 2) ? cw[b][0].x : cw[b][0].y;
            const uint32_t w1 = (s < 2) ? cw[b][1].x : cw[b][1].y;
            af[b][0] = lds_u32(__byte_perm(w0, laneword, 0x7604u | (p0 << 4)));
            af[b][1] = lds_u32(__byte_perm(w1, laneword, 0x7604u | (p0 << 4)));
            af[b][2] = lds_u32(__byte_perm(w0, laneword, 0x7604u | (p1 << 4)));
            af[b][3] = lds_u32(__byte_perm(w1, laneword, 0x7604u | (p1 << 4)));
          }
#pragma unroll
          for (int b = 0; b < BG; ++b)
#pragma unroll
            for (int ng = 0; ng < NG; ++ng)
              mma_16816_f16_nv(acc[b][ng], af[b][0], af[b][1], af[b][2], af[b][3], xf[jg + b][s][ng][0],
                               xf[jg + b][s][ng][1]);
        }
#pragma unroll
        for (int b = 0; b < BG; ++b)
#pragma unroll
          for (int ng = 0; ng < NG; ++ng) {
            part[ng][0] = fmaf(S4[0][jg + b], acc[b][ng][0], part[ng][0]);
            part[ng][1] = fmaf(S4[0][jg + b], acc[b][ng][1], part[ng][1]);
            part[ng][2] = fmaf(S4[1][jg + b], acc[b][ng][2], part[ng][2]);
            part[ng][3] = fmaf(S4[1][jg + b], acc[b][ng][3], part[ng][3]);
          }
      }
    }
    // partials, unscaled to true units, into this unit's slot (no barrier)
    if (active) {
      float *rb = red + (fs * kDecWarps + warp) * 17 * TR;
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const int t = 2 * q + 8 * ng;
        *reinterpret_cast<float2 *>(rb + g * TR + t) =
            make_float2(part[ng][0] * unscale[ng][0], part[ng][1] * unscale[ng][1]);
        *reinterpret_cast<float2 *>(rb + (g + 8) * TR + t) =
            make_float2(part[ng][2] * unscale[ng][0], part[ng][3] * unscale[ng][1]);
      }
    }
    // This warp is done with the slot: the store above waited for this lane's
    // last MMA of the unit, and an MMA completes only once every lane of the warp
    // has supplied its operands, so every lane's reads of the slot are done.  The
    // warp that finishes the slot last refills it with unit i + S.
    if (active && landed && lane == 0) {
      const uint32_t old = atomicAdd(ecnt + slot, 1u);
      if (old == static_cast<uint32_t>((ring_round + 1) * nact - 1) && i + S < nu) load_unit(i + S);
    }
    // the s*T entries' copy, once the rank CTAs have had the time to publish them
    if (tid == 0 && i == (nu >= 2 ? nu - 2 : 0)) {
      ptx::mbar_arrive_expect_tx(tbar, a.stf_bytes);
      ptx::bulk_g2s(const_cast<uint64_t *>(stf_s), a.stf_g, a.stf_bytes, tbar);
    }
    if (fs == F - 1 || i + 1 == nu) {
      // round end: unit i - fs + f sits in slot f.  Warp w sums row w of every
      // row group (its warp slices in a fixed order) into yacc.
      __syncthreads();
      const int tc = lane % TR, pw = lane / TR;
      for (int f = 0; f <= fs; ++f) {
        const int u = i - fs + f;
        for (int rs = 0; rs < RPS; ++rs) {
          const float *rb = red + ((f * kDecWarps + rs * WPR) * 17 + warp) * TR;
          float v = 0.0f;
          for (int w = pw; w < WPR; w += 32 / TR) v += rb[w * 17 * TR + tc];
#pragma unroll
          for (int o = TR; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane < TR) yacc[(u * rows_per_unit + 16 * rs + warp) * TR + tc] = v;
        }
      }
      __syncthreads();  // yacc complete, slots free
      fs = 0;
    } else {
      ++fs;
    }
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
      ++ring_round;
    }
    sfp += unit_sf;
    rows_left -= rows_per_unit;
  }

  // ---- grid generation: the last arrival resets the count and advances it
  if (tid == 0) {
    if (arrive_old == static_cast<uint32_t>(a.G) - 1u) {
      ptx::st_relaxed_gpu(a.bar_count, 0u);
      ptx::st_relaxed_gpu(a.bar_gen, gen_next);
    } else if (arrive_old >= static_cast<uint32_t>(a.G)) {
      raise_status(a.status, QLORA_ERR_TIMEOUT);  // the header was not zeroed
    }
  }

  // ---- tail: s*T entries of this call (copied again until every tag matches),
  // then the LoRA term of every row group, added to the reduced sums and stored
  // (every decision below is made by all threads together: the barriers stay uniform)
  bool have_t = __syncthreads_and(flags[1] == 0 && ptx::mbar_wait(tbar, 0, abort_flag) &&
                                  ptx::mbar_wait(bbar, 0, abort_flag));
  const int nkk = r16 >> 4;
  const int tcheck = nkk * NG * 32 * 4;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t phase = 0; have_t; ++phase) {
    bool mine = true;
    for (int e = tid; e < tcheck; e += kDecThreads) {
      const int ln = (e >> 2) & 31, ng = (e >> 7) % NG;
      const int t = (ln >> 2) + 8 * ng;
      if (t < a.M) mine = mine && static_cast<uint32_t>(stf_s[e] >> 32) == tag;
    }
    if (__syncthreads_and(mine)) break;
    if (__syncthreads_or(tid == 0 && ptx::globaltimer_ns() - t0 > ptx::kWaitNs)) {
      have_t = false;
      break;
    }
    if (tid == 0) {  // the previous copy has completed (phase) and been read: copy again
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive_expect_tx(tbar, a.stf_bytes);
      ptx::bulk_g2s(const_cast<uint64_t *>(stf_s), a.stf_g, a.stf_bytes, tbar);
    }
    have_t = __syncthreads_and(ptx::mbar_wait(tbar, (phase + 1) & 1, nullptr));
  }
  if (!have_t) {
    if (tid == 0) raise_status(a.status, QLORA_ERR_TIMEOUT);
    return;
  }
  auto store_y = [&](int64_t n, int t, float v) {
    if (a.y_f32) reinterpret_cast<float *>(a.Y)[static_cast<int64_t>(t) * a.N + n] = v;
    else reinterpret_cast<__nv_bfloat16 *>(a.Y)[static_cast<int64_t>(t) * a.N + n] = __float2bfloat16_rn(v);
  };
  // task k (unit k / RPS, row group k % RPS) by warp k % 16: D = (B rows)(s T)^T
  // on tensor cores (bf16), rows g / g + 8, tokens 2q, 2q + 1 (+ 8 ng)
  const int ntask = nu * RPS;
  for (int k = warp; k < ntask; k += kDecWarps) {
    const int i = k / RPS, rs = k % RPS;
    float d[NG][4];
#pragma unroll
    for (int ng = 0; ng < NG; ++ng) d[ng][0] = d[ng][1] = d[ng][2] = d[ng][3] = 0.0f;
    const int row0 = 16 * rs + g;  // row within the unit
    for (int kk = 0; kk < nkk; ++kk) {
      const uint8_t *r0 = at(Lay.brows) + i * a.brow_unit_bytes + ((kk >> 2) * rows_per_unit + row0) * 128;
      const uint8_t *r1 = r0 + 8 * 128;
      const uint32_t u0 = ((2 * (kk & 3)) ^ g) << 4, u1 = ((2 * (kk & 3) + 1) ^ g) << 4;
      const uint32_t a0 = *reinterpret_cast<const uint32_t *>(r0 + u0 + 4 * q);
      const uint32_t a1 = *reinterpret_cast<const uint32_t *>(r1 + u0 + 4 * q);
      const uint32_t a2 = *reinterpret_cast<const uint32_t *>(r0 + u1 + 4 * q);
      const uint32_t a3 = *reinterpret_cast<const uint32_t *>(r1 + u1 + 4 * q);
#pragma unroll
      for (int ng = 0; ng < NG; ++ng) {
        const uint64_t *en = stf_s + ((kk * NG + ng) * 32 + lane) * 4;
        const uint32_t b0 = static_cast<uint32_t>(en[0] & 0xffffu) | (static_cast<uint32_t>(en[1] & 0xffffu) << 16);
        const uint32_t b1 = static_cast<uint32_t>(en[2] & 0xffffu) | (static_cast<uint32_t>(en[3] & 0xffffu) << 16);
        mma_16816(d[ng], a0, a1, a2, a3, b0, b1);
      }
    }
    const int64_t n0 = static_cast<int64_t>(U0 + i) * rows_per_unit + 16 * rs;
#pragma unroll
    for (int ng = 0; ng < NG; ++ng)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rr = g + 8 * (e >> 1), t = 2 * q + (e & 1) + 8 * ng;
        const int64_t n = n0 + rr;
        if (t < a.M && n < a.N) store_y(n, t, yacc[(i * rows_per_unit + 16 * rs + rr) * TR + t] + d[ng][e]);
      }
  }
}

// Start of the dynamic shared-memory window (after the block's reservation).
inline uint32_t decode_smem_base(int dev) { return dyn_smem_base(dev); }

inline qlora_status launch_decode(const DecodePlan &p, const DecodeArgs &args, const CUtensorMap &tm_codes,
                                  const CUtensorMap &tm_b, int dev, cudaStream_t st) {
  static std::once_flag flags[2][64];
  static qlora_status results[2][64];
  const int which = p.NG == 2 ? 1 : 0;
  auto kernel = p.NG == 2 ? nf4_decode_kernel<2> : nf4_decode_kernel<1>;
  std::call_once(flags[which][dev], [&] {
    results[which][dev] =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDecSmemLimit)) ==
                cudaSuccess
            ? QLORA_OK
            : QLORA_ERR_CUDA;
    cudaGetLastError();
  });
  if (results[which][dev] != QLORA_OK) return results[which][dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.G);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = p.dyn_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, tm_codes, tm_b, args, p.dyn_bytes) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

}  // namespace qlora
