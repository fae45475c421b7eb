// Persistent warp-specialised tcgen05 GEMM for sm_100a, with an NF4-dequantising
// producer for the frozen weight operand and the rank-r LoRA product folded in as
// extra K steps of the same accumulator.
//
//   D[M_rows, N_cols] = A (.) B^T  (+ A2 (.) B2^T)      fp32 accumulate in TMEM
//
// Operands are bf16 in 128-byte-swizzled shared memory.  A is always loaded by TMA
// (K-major or MN-major); B is either loaded by TMA or produced by 8 "dequant"
// warps from packed NF4 codes (TMA-staged) and the E4M3 block scales:
//   w' = bf16_rne(fl32(L[code] * fl32(E4M3(q) * c2)))
// exactly the dequantised weight of the glossary page's forward rule ("How QLoRA
// works": dequantise to bfloat16 right before the matmul).  The forward pass uses
// W' as a K-major B operand (rows = out features); the backward dX pass uses the
// same tile as an MN-major B operand (rows = in features), so one decode routine
// serves both.
//
// Roles (warp index):  0 TMA producer | 1 MMA issuer + TMEM owner |
//                      4..7 epilogue (TMEM lane quadrants 0..3) | 8..15 dequant.
// Every wait is bounded; a wait that gives up raises QLORA_ERR_TIMEOUT in the
// status word, sets a CTA abort flag so the other roles leave too, drains the
// copies and MMAs this CTA has in flight (again bounded) and frees TMEM.
#pragma once

#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

struct GemmArgs {
  int M_rows;        // rows of D (tiles of 128 * MT)
  int N_cols;        // cols of D (tiles of BN)
  int k_steps;       // main K steps of 64
  int hilo_cols;     // 1: a tile's B holds BN/2 columns of B (tmB) then the same
                     //    columns of B2 (tmB2); D columns j and j + BN/2 are summed
  int ksplit;        // K range split over this many CTAs (non-NF4, no LoRA steps); > 1
                     // writes raw fp32 partial planes to `part` [ksplit][M_rows][N_cols]
  float *part;
  int k_per;         // K steps per split when ksplit > 1 (no split is empty)
  // masked accumulate (non-transposed `out` only): out += v * out_scale * (keep bit ? keep_scale : 0),
  // keep = [M_rows][N_cols / 8] bits, bit (col % 8) of byte col / 8
  const uint8_t *keep;
  float keep_scale;
  int lora_steps;    // extra K steps of 64 for the LoRA block (0 = none)
  int lora_r;        // LoRA rank (bounds the B2 rows/cols read by the dequant warps)
  // outputs (each optional): `out` (f32 or bf16, scaled by out_scale, optionally
  // transposed) and a bf16 pair hi = bf16(v * hl_scale), lo = bf16(v * hl_scale - hi)
  void *out;
  int64_t ldo;
  int out_f32;       // 1: float32, 0: bf16
  int out_transpose; // 1: out[col * ldo + row]
  float out_scale;
  __nv_bfloat16 *out_hi;
  __nv_bfloat16 *out_lo;
  int64_t ld_hl;
  float hl_scale;
  // NF4 operand (B from dequant)
  const uint8_t *scale_codes;
  const float *c2;
  int scale_format;  // qlora_scale_format of scale_codes
  int64_t w_rows;    // N of W
  int64_t w_cols;    // K of W
  const __nv_bfloat16 *lora_b2;  // B2 source read by the dequant warps (fwd: B [N, r]; bwd: A [r, K])
  int64_t lora_ld;   // row stride of lora_b2 (elements)
  uint32_t *status;
};

template <bool A_MN, bool B_MN, bool NF4, int BN, int MT>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int A_STAGE = MT * BM * BK * 2;
  static constexpr int B_STAGE = BN * BK * 2;
  static constexpr int C_STAGE = NF4 ? BN * 32 : 0;  // codes: 64 weights (32 B) per B row
  static constexpr int SA = NF4 ? (MT == 1 ? 4 : 3) : 6;
  static constexpr int SB = NF4 ? 3 : SA;
  static constexpr int SC = NF4 ? 4 : 1;
  static constexpr int NUM_ACC = (2 * MT * BN <= 512) ? 2 : 1;
  static constexpr int ACC_COLS = MT * BN;
  static constexpr int TMEM_COLS = (NUM_ACC * ACC_COLS <= 32) ? 32 : (NUM_ACC * ACC_COLS <= 64) ? 64
                                   : (NUM_ACC * ACC_COLS <= 128) ? 128 : (NUM_ACC * ACC_COLS <= 256) ? 256 : 512;
  static constexpr int THREADS = NF4 ? 512 : 256;
  static constexpr int SMEM_DATA = SA * A_STAGE + SB * B_STAGE + SC * C_STAGE;
  static constexpr int SMEM_BYTES = SMEM_DATA + 1024 /*align*/ + 512 /*barriers*/;
  static constexpr uint32_t IDESC = ptx::idesc_bf16(BM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
  static_assert(BN % 64 == 0 || (!NF4 && BN >= 16), "tile");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Byte offset of the 16-byte chunk `c` (0..7) of the 128-byte row `row` inside a
// 1024-byte SW128 atom.
__device__ __forceinline__ uint32_t sw128_row_chunk(uint32_t row, uint32_t c) {
  return (row & 7u) * 128u + ((c ^ (row & 7u)) << 4);
}

// Table of the 16 products bf16(L[c] * S) of one block, split into byte planes:
// lo[j] / hi[j] hold the low / high bytes of entries 4j .. 4j + 3.
__device__ __forceinline__ void nf4_planes(float S, uint32_t (&lo)[4], uint32_t (&hi)[4]) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(__fmul_rn(nf4_level(2 * j), S), __fmul_rn(nf4_level(2 * j + 1), S));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    lo[j] = __byte_perm(p[2 * j], p[2 * j + 1], 0x6420);
    hi[j] = __byte_perm(p[2 * j], p[2 * j + 1], 0x7531);
  }
}

// The eight codes of one 32-bit word (low nibble first) -> four packed bf16x2
// words o[0..3] (code 2i in the low half of o[i]), looked up in the byte planes
// with byte permutes: the low three bits of a code pick an entry in each half of
// the table, the fourth bit picks the half.
__device__ __forceinline__ void nf4_word(uint32_t w, const uint32_t (&lo)[4], const uint32_t (&hi)[4], uint32_t *o) {
  const uint32_t sel32 = w & 0x77777777u;
  const uint32_t msel32 = 0x32103210u | ((w >> 1) & 0x44444444u);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sel = h ? (sel32 >> 16) : sel32;
    const uint32_t msel = h ? (msel32 >> 16) : msel32;
    const uint32_t la = __byte_perm(lo[0], lo[1], sel), lb = __byte_perm(lo[2], lo[3], sel);
    const uint32_t ha = __byte_perm(hi[0], hi[1], sel), hb = __byte_perm(hi[2], hi[3], sel);
    const uint32_t l = __byte_perm(la, lb, msel), hh = __byte_perm(ha, hb, msel);
    o[h * 2 + 0] = __byte_perm(l, hh, 0x5140);
    o[h * 2 + 1] = __byte_perm(l, hh, 0x7362);
  }
}

// Decode 64 NF4 codes (two uint4 of packed nibbles) with block scale S into 32
// packed bf16x2 words.
__device__ __forceinline__ void nf4_decode64(const uint4 &c0, const uint4 &c1, float S, uint32_t (&o)[32]) {
  uint32_t lo[4], hi[4];
  nf4_planes(S, lo, hi);
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int q = 0; q < 8; ++q) nf4_word(w[q], lo, hi, o + 4 * q);
}

__device__ __forceinline__ void store_row128(uint8_t *atom_base, uint32_t row, const uint32_t (&o)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    *reinterpret_cast<uint4 *>(atom_base + sw128_row_chunk(row, c)) =
        make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
  }
}

// 64 bf16 (128 bytes) from global, zero where col >= ncols or !valid.
__device__ __forceinline__ void load_row128(const __nv_bfloat16 *src, int valid_cols, uint32_t (&o)[32]) {
  if (valid_cols >= 64) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = __ldg(s + c);
      o[4 * c] = v.x; o[4 * c + 1] = v.y; o[4 * c + 2] = v.z; o[4 * c + 3] = v.w;
    }
  } else {
    const uint16_t *s = reinterpret_cast<const uint16_t *>(src);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t a = (2 * i < valid_cols) ? __ldg(s + 2 * i) : 0u;
      const uint32_t b = (2 * i + 1 < valid_cols) ? __ldg(s + 2 * i + 1) : 0u;
      o[i] = a | (b << 16);
    }
  }
}

constexpr int kGemmDequantThreads = 256;  // NF4 producer threads (warps 8..15)

// out[row, col0 + j] += v_j * out_scale * (keep bit ? keep_scale : 0), j < ncol.
__device__ __forceinline__ void masked_accumulate32(const GemmArgs &args, int row, int col0, int ncol,
                                                 const uint32_t (&v)[32]) {
  const uint8_t *kp = args.keep + (int64_t)row * (args.N_cols / 8) + col0 / 8;
  uint32_t bits = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b)
    if (8 * b < ncol) bits |= static_cast<uint32_t>(kp[b]) << (8 * b);
  if (args.out_f32) {
    float *o = reinterpret_cast<float *>(args.out) + (int64_t)row * args.ldo + col0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < ncol && ((bits >> j) & 1u)) o[j] += __uint_as_float(v[j]) * args.out_scale * args.keep_scale;
  } else {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(args.out) + (int64_t)row * args.ldo + col0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < ncol && ((bits >> j) & 1u))
        o[j] = __float2bfloat16_rn(__bfloat162float(o[j]) +
                                   __uint_as_float(v[j]) * args.out_scale * args.keep_scale);
  }
}

// Stores one 32-column chunk of accumulator row `row` (v = fp32 bit patterns).
__device__ __forceinline__ void store_chunk32(const GemmArgs &args, int row, int col0, int ncol,
                                              const uint32_t (&v)[32]) {
  if (args.keep) {
    masked_accumulate32(args, row, col0, ncol, v);
    return;
  }
  const bool full = ncol == 32;
  if (args.out) {
    if (!args.out_transpose) {
      if (args.out_f32) {
        float *o = reinterpret_cast<float *>(args.out) + (int64_t)row * args.ldo + col0;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 f = make_float4(__uint_as_float(v[j]) * args.out_scale, __uint_as_float(v[j + 1]) * args.out_scale,
                                       __uint_as_float(v[j + 2]) * args.out_scale,
                                       __uint_as_float(v[j + 3]) * args.out_scale);
          if (full) {
            *reinterpret_cast<float4 *>(o + j) = f;
          } else {
            if (j < ncol) o[j] = f.x;
            if (j + 1 < ncol) o[j + 1] = f.y;
            if (j + 2 < ncol) o[j + 2] = f.z;
            if (j + 3 < ncol) o[j + 3] = f.w;
          }
        }
      } else {
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(args.out) + (int64_t)row * args.ldo + col0;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[j + 2 * i]) * args.out_scale,
                                __uint_as_float(v[j + 2 * i + 1]) * args.out_scale);
          if (full) {
            *reinterpret_cast<uint4 *>(o + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          } else {
            uint16_t *o16 = reinterpret_cast<uint16_t *>(o);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (j + i < ncol) o16[j + i] = (i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xffffu);
          }
        }
      }
    } else {
      // out[col * ldo + row]: lanes write consecutive rows of each column.
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < ncol) {
          const float x = __uint_as_float(v[j]) * args.out_scale;
          if (args.out_f32) reinterpret_cast<float *>(args.out)[(int64_t)(col0 + j) * args.ldo + row] = x;
          else reinterpret_cast<__nv_bfloat16 *>(args.out)[(int64_t)(col0 + j) * args.ldo + row] = __float2bfloat16_rn(x);
        }
      }
    }
  }
  if (args.out_hi) {
    uint16_t *oh = reinterpret_cast<uint16_t *>(args.out_hi) + (int64_t)row * args.ld_hl + col0;
    uint16_t *ol = reinterpret_cast<uint16_t *>(args.out_lo) + (int64_t)row * args.ld_hl + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint32_t h[4], l[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(v[j + 2 * i]) * args.hl_scale;
        const float b = __uint_as_float(v[j + 2 * i + 1]) * args.hl_scale;
        h[i] = pack_bf16x2(a, b);
        l[i] = pack_bf16x2(a - bf16lo_to_f32(h[i]), b - bf16hi_to_f32(h[i]));
      }
      if (full) {
        *reinterpret_cast<uint4 *>(oh + j) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(ol + j) = make_uint4(l[0], l[1], l[2], l[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (j + i < ncol) {
            oh[j + i] = (i & 1) ? (h[i >> 1] >> 16) : (h[i >> 1] & 0xffffu);
            ol[j + i] = (i & 1) ? (l[i >> 1] >> 16) : (l[i >> 1] & 0xffffu);
          }
        }
      }
    }
  }
}

// Sums the ksplit fp32 partial planes of a split-K GEMM in plane order and
// writes the outputs exactly as the GEMM epilogue does (out = v * out_scale;
// hi = bf16(v * hl_scale), lo = bf16(v * hl_scale - hi)).  Two columns per thread.
__global__ void splitk_finish_kernel(const GemmArgs args) {
  ptx::griddep_launch();
  ptx::griddep_wait();  // the partial planes are complete
  const int64_t pairs = (int64_t)args.M_rows * args.N_cols / 2;
  const int64_t plane = (int64_t)args.M_rows * args.N_cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < pairs; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = 2 * i;
    float a = 0.0f, b = 0.0f;
    for (int sp = 0; sp < args.ksplit; ++sp) {
      const float2 p = *reinterpret_cast<const float2 *>(args.part + sp * plane + e);
      a += p.x;
      b += p.y;
    }
    const int64_t row = e / args.N_cols, col = e - row * args.N_cols;
    if (args.out) {
      if (args.out_f32) {
        float *o = reinterpret_cast<float *>(args.out) + row * args.ldo + col;
        o[0] = a * args.out_scale;
        o[1] = b * args.out_scale;
      } else {
        *reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(args.out) + row * args.ldo + col) =
            pack_bf16x2(a * args.out_scale, b * args.out_scale);
      }
    }
    if (args.out_hi) {
      const float x = a * args.hl_scale, y = b * args.hl_scale;
      const uint32_t h = pack_bf16x2(x, y);
      const uint32_t l = pack_bf16x2(x - bf16lo_to_f32(h), y - bf16hi_to_f32(h));
      *reinterpret_cast<uint32_t *>(args.out_hi + row * args.ld_hl + col) = h;
      *reinterpret_cast<uint32_t *>(args.out_lo + row * args.ld_hl + col) = l;
    }
  }
}

template <bool A_MN, bool B_MN, bool NF4, int BN, int MT>
__global__ void __launch_bounds__(GemmCfg<A_MN, B_MN, NF4, BN, MT>::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
               const __grid_constant__ CUtensorMap tmCodes, const GemmArgs args,
               const __grid_constant__ CUtensorMap tmAg, const __grid_constant__ CUtensorMap tmBg,
               const __grid_constant__ CUtensorMap tmB2g, const GemmArgs argsg) {
  using C = GemmCfg<A_MN, B_MN, NF4, BN, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + C::SA * C::A_STAGE;
  uint8_t *sC = sB + C::SB * C::B_STAGE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sC + C::SC * C::C_STAGE);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + C::SA;
  uint64_t *full_b = empty_a + C::SA;
  uint64_t *empty_b = full_b + C::SB;
  uint64_t *full_c = empty_b + C::SB;
  uint64_t *empty_c = full_c + C::SC;
  uint64_t *acc_full = empty_c + C::SC;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SA; ++s) { ptx::mbar_init(&full_a[s], 1); ptx::mbar_init(&empty_a[s], 1); }
    for (int s = 0; s < C::SB; ++s) {
      ptx::mbar_init(&full_b[s], NF4 ? kGemmDequantThreads : 1);
      ptx::mbar_init(&empty_b[s], 1);
    }
    for (int s = 0; s < C::SC; ++s) { ptx::mbar_init(&full_c[s], 1); ptx::mbar_init(&empty_c[s], kGemmDequantThreads); }
    for (int s = 0; s < 2; ++s) { ptx::mbar_init(&acc_full[s], 1); ptx::mbar_init(&acc_empty[s], 4); }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    if (!NF4) ptx::prefetch_tmap(&tmB);
    if (args.hilo_cols) ptx::prefetch_tmap(&tmB2);
    if (args.lora_steps) ptx::prefetch_tmap(&tmA2);
    if (NF4) ptx::prefetch_tmap(&tmCodes);
    if (argsg.M_rows > 0) {
      ptx::prefetch_tmap(&tmAg);
      ptx::prefetch_tmap(&tmBg);
      if (args.hilo_cols) ptx::prefetch_tmap(&tmB2g);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above overlaps the preceding kernel's tail; every global read and
  // write below comes after that kernel has completed.
  ptx::griddep_launch();
  ptx::griddep_wait();

  const int tile_n = args.hilo_cols ? BN / 2 : BN;  // output columns per tile
  const int num_m = (args.M_rows + C::BM * MT - 1) / (C::BM * MT);
  const int num_n = (args.N_cols + tile_n - 1) / tile_n;
  const int tiles_mn = num_m * num_n;
  const int ksplit = args.ksplit > 1 ? args.ksplit : 1;
  const int num_tiles1 = tiles_mn * ksplit;
  // A second, independent problem (argsg: its own maps, output and sizes; the
  // same tile shape and column halves, no K split and no LoRA steps) may share
  // the launch: its tiles follow this one's, so both run at once.
  const int num_m_g = argsg.M_rows > 0 ? (argsg.M_rows + C::BM * MT - 1) / (C::BM * MT) : 0;
  const int num_n_g = argsg.M_rows > 0 ? (argsg.N_cols + tile_n - 1) / tile_n : 0;
  const int num_tiles = num_tiles1 + num_m_g * num_n_g;
  auto tile_of = [&](int w, int &m0, int &n0) {
    if (w >= num_tiles1) {
      const int v = w - num_tiles1;
      m0 = (v % num_m_g) * C::BM * MT;
      n0 = (v / num_m_g) * tile_n;
      return;
    }
    const int mn = w % tiles_mn;
    m0 = (mn % num_m) * C::BM * MT;
    n0 = (mn / num_m) * tile_n;
  };
  const int main_steps = args.k_steps;
  const int steps = main_steps + args.lora_steps;
  // main (non-LoRA) K steps of tile w's problem
  auto main_of = [&](int w) { return w >= num_tiles1 ? argsg.k_steps : main_steps; };
  // K steps [k_begin, k_end) of tile w (its share of the split)
  const int k_per = ksplit > 1 ? args.k_per : steps;
  auto k_range = [&](int w, int &kb, int &ke) {
    if (w >= num_tiles1) {
      kb = 0;
      ke = argsg.k_steps;
      return;
    }
    const int sp = w / tiles_mn;
    kb = sp * k_per;
    ke = min(steps, kb + k_per);
  };

  auto fail = [&]() {
    raise_status(args.status, QLORA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (ptx::elect_one()) {
      uint32_t sa = 0, pa = 0, sc = 0, pc = 0;
      int issued_a = 0, issued_c = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int m0, n0, kb, ke;
        tile_of(tile, m0, n0);
        k_range(tile, kb, ke);
        const bool g2 = tile >= num_tiles1;
        const CUtensorMap *mA = g2 ? &tmAg : &tmA, *mB = g2 ? &tmBg : &tmB, *mB2 = g2 ? &tmB2g : &tmB2;
        const int ms = main_of(tile);
        for (int ks = kb; ks < ke && ok; ++ks) {
          const bool lora = ks >= ms;
          const int kk = ks;
          if (NF4 && !lora) {
            if (!ptx::mbar_wait(&empty_c[sc], pc ^ 1, abort_flag)) { ok = false; break; }
            ptx::mbar_arrive_expect_tx(&full_c[sc], C::C_STAGE);
            // fwd: rows n0.., 32 code bytes of K step ks; bwd: 64 rows of W, BN/2 code bytes
            if (!B_MN) ptx::tma_load_2d(sC + sc * C::C_STAGE, &tmCodes, &full_c[sc], ks * 32, n0);
            else ptx::tma_load_2d(sC + sc * C::C_STAGE, &tmCodes, &full_c[sc], n0 / 2, ks * 64);
            ++issued_c;
            if (++sc == C::SC) { sc = 0; pc ^= 1; }
          }
          if (!ptx::mbar_wait(&empty_a[sa], pa ^ 1, abort_flag)) { ok = false; break; }
          const uint32_t bytes = C::A_STAGE + (NF4 ? 0 : C::B_STAGE);
          ptx::mbar_arrive_expect_tx(&full_a[sa], bytes);
          uint8_t *dA = sA + sa * C::A_STAGE;
          if (lora) {
            const int k2 = (ks - main_steps) * 64;
            for (int t = 0; t < MT; ++t) ptx::tma_load_2d(dA + t * 16384, &tmA2, &full_a[sa], k2, m0 + t * 128);
          } else if (!A_MN) {
            for (int t = 0; t < MT; ++t) ptx::tma_load_2d(dA + t * 16384, mA, &full_a[sa], kk * 64, m0 + t * 128);
          } else {
            for (int t = 0; t < MT * 2; ++t) ptx::tma_load_2d(dA + t * 8192, mA, &full_a[sa], m0 + t * 64, kk * 64);
          }
          if (!NF4) {
            uint8_t *dB = sB + sa * C::B_STAGE;
            if (!B_MN) {
              ptx::tma_load_2d(dB, mB, &full_a[sa], kk * 64, n0);
            } else if (!args.hilo_cols) {
              for (int t = 0; t < BN / 64; ++t) ptx::tma_load_2d(dB + t * 8192, mB, &full_a[sa], n0 + t * 64, kk * 64);
            } else {  // columns n0.. of B, then the same columns of B2
              constexpr int kHalfBlocks = BN >= 128 ? BN / 128 : 1;  // 64-column blocks per half
              for (int t = 0; t < BN / 64; ++t) {
                const int h = t / kHalfBlocks;
                ptx::tma_load_2d(dB + t * 8192, h ? mB2 : mB, &full_a[sa], n0 + (t % kHalfBlocks) * 64, kk * 64);
              }
            }
          }
          ++issued_a;
          if (++sa == C::SA) { sa = 0; pa ^= 1; }
        }
      }
      if (!ok) fail();
      // Drain: the last (up to) SA / SC copies issued must have landed before the
      // CTA may exit (older ones were consumed already).
      for (int i = 0; i < C::SA && i < issued_a; ++i) {
        if (sa == 0) { sa = C::SA - 1; pa ^= 1; } else { --sa; }
        ptx::mbar_wait(&full_a[sa], pa, nullptr);
      }
      for (int i = 0; NF4 && i < C::SC && i < issued_c; ++i) {
        if (sc == 0) { sc = C::SC - 1; pc ^= 1; } else { --sc; }
        ptx::mbar_wait(&full_c[sc], pc, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (ptx::elect_one()) {
      uint32_t sa = 0, pa = 0, sb = 0, pb = 0;
      int it = 0;
      bool ok = true;
      const uint32_t sA0 = ptx::smem_addr(sA), sB0 = ptx::smem_addr(sB);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it % C::NUM_ACC;
        const uint32_t acc_phase = (it / C::NUM_ACC) & 1;
        int kb, ke;
        k_range(tile, kb, ke);
        const int ms = main_of(tile);
        if (!ptx::mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
        for (int ks = kb; ks < ke && ok; ++ks) {
          const bool lora = ks >= ms;
          if (!ptx::mbar_wait(&full_a[sa], pa, abort_flag)) { ok = false; break; }
          if (NF4 && !ptx::mbar_wait(&full_b[sb], pb, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a_base = sA0 + sa * C::A_STAGE;
          const uint32_t b_base = sB0 + (NF4 ? sb : sa) * C::B_STAGE;
          const bool a_mn = A_MN && !lora;  // the LoRA A2 block is K-major
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_base + k16 * 2048, 8192, 1024)
                                     : ptx::smem_desc_sw128(b_base + k16 * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const uint64_t ad = a_mn ? ptx::smem_desc_sw128(a_base + t * 16384 + k16 * 2048, 8192, 1024)
                                       : ptx::smem_desc_sw128(a_base + t * 16384 + k16 * 32, 16, 1024);
              const uint32_t idesc = a_mn ? C::IDESC : (C::IDESC & ~(1u << 15));
              ptx::mma_bf16(d_tmem + t * BN, ad, bd, idesc, (ks != kb || k16) ? 1u : 0u);
            }
          }
          ptx::mma_commit(&empty_a[sa]);
          if (NF4) ptx::mma_commit(&empty_b[sb]);
          if (++sa == C::SA) { sa = 0; pa ^= 1; }
          if (NF4 && ++sb == C::SB) { sb = 0; pb ^= 1; }
        }
        if (ok) ptx::mma_commit(&acc_full[acc]);
      }
      if (!ok) fail();
      // Wait until every MMA this thread issued has completed.
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;  // TMEM lane quadrant (warp % 4)
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it % C::NUM_ACC;
      const uint32_t acc_phase = (it / C::NUM_ACC) & 1;
      if (!ptx::mbar_wait(&acc_full[acc], acc_phase, abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      ptx::tc_fence_after();
      int m0, n0;
      tile_of(tile, m0, n0);
      const bool g2 = tile >= num_tiles1;
      const GemmArgs &ea = g2 ? argsg : args;  // the tile's problem
      const int sp = g2 ? 0 : tile / tiles_mn;
      for (int t = 0; t < MT; ++t) {
        const int row = m0 + t * 128 + q * 32 + lane;
        for (int cb = 0; cb < tile_n; cb += 32) {
          uint32_t v[32];
          const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS + t * BN + cb;
          ptx::tmem_ld32(taddr, v);
          ptx::tmem_ld_wait();
          if (args.hilo_cols) {  // add the B2 half of the tile
            uint32_t w2[32];
            ptx::tmem_ld32(taddr + BN / 2, w2);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(w2[j]));
          }
          const int col0 = n0 + cb;
          if (row < ea.M_rows && col0 < ea.N_cols) {
            if (ksplit > 1 && !g2) {  // raw fp32 partial of this K share
              float *o = args.part + ((int64_t)sp * args.M_rows + row) * args.N_cols + col0;
              const int nc = min(32, args.N_cols - col0);
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nc) o[j] = __uint_as_float(v[j]);
            } else {
              store_chunk32(ea, row, col0, min(32, ea.N_cols - col0), v);
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[acc]);
    }
  } else if (NF4 && warp >= 8) {
    // ------------------------------------------------------------ dequant producer
    const int d = threadIdx.x - 256;  // 0..255
    const int64_t kblocks = args.w_cols / 64;
    // Thread -> (B row it fills, code bytes it reads).  Chosen so that, within
    // every quarter-warp, the eight 16-byte code reads and the eight swizzled
    // 16-byte operand writes each fall on distinct banks.
    int wr, fb;                // fwd: W row n0 + wr; dX: W row ks*64 + wr, in-feature block fb
    uint32_t atom_off, row_in, code_off, half_first;
    if (!B_MN) {
      wr = d;
      fb = 0;
      atom_off = (d >> 3) * 1024;
      row_in = d & 7;
      code_off = d * 32;
      half_first = (d >> 2) & 1;
    } else {
      const int P = d >> 3, j = d & 7;
      wr = 8 * (P & 7) + j;                  // 0..63: W row within the K step
      fb = ((j >> 1) + (P >> 3)) & 3;        // 64-feature block within the tile
      atom_off = fb * 8192 + (wr >> 3) * 1024;
      row_in = wr & 7;
      code_off = wr * 128 + fb * 32;
      half_first = j & 1;
    }
    // Block scale (E4M3 byte, c2) of flat step (tile, ks), loaded two steps
    // before use into one of two register slots that are only ever refilled
    // after being consumed.
    auto scale_src = [&](int tile, int ks, uint32_t &qv, float &cv) {
      qv = 0x100u;  // "no block": rows past N, LoRA steps, past the last tile
      cv = 0.0f;
      if (tile >= num_tiles || ks >= main_steps) return;
      int m0_, n0;
      tile_of(tile, m0_, n0);
      int64_t wrow, kblk;
      if (!B_MN) { wrow = n0 + wr; kblk = ks; }
      else { wrow = (int64_t)ks * 64 + wr; kblk = n0 / 64 + fb; }
      if (wrow < args.w_rows && kblk < kblocks) {
        const int64_t b = wrow * kblocks + kblk;
        qv = __ldg(args.scale_codes + b);
        cv = __ldg(args.c2 + (b >> 8));
      }
    };
    uint32_t sb = 0, pb = 0, sc = 0, pc = 0;
    bool ok = true;
    int tile = blockIdx.x, ks = 0;        // step being produced
    int ptile = blockIdx.x, pks = 0;      // step whose scale is fetched next
    auto advance = [&](int &t, int &k) {
      if (++k == steps) { k = 0; t += gridDim.x; }
    };
    uint32_t qa, qb;
    float ca, cb;
    scale_src(ptile, pks, qa, ca);
    advance(ptile, pks);
    scale_src(ptile, pks, qb, cb);
    advance(ptile, pks);

    auto produce = [&](uint32_t &qs, float &cs) -> bool {
      const bool lora = ks >= main_steps;
      int m0_, n0;
      tile_of(tile, m0_, n0);
      uint32_t o[32];
      if (!lora) {
        if (!ptx::mbar_wait(&full_c[sc], pc, abort_flag)) return false;
        const uint8_t *csrc = sC + sc * C::C_STAGE + code_off;
        const uint4 x0 = *reinterpret_cast<const uint4 *>(csrc + 16 * half_first);
        const uint4 x1 = *reinterpret_cast<const uint4 *>(csrc + 16 * (1 - half_first));
        ptx::mbar_arrive(&empty_c[sc]);
        if (++sc == C::SC) { sc = 0; pc ^= 1; }
        const uint4 c0 = half_first ? x1 : x0, c1 = half_first ? x0 : x1;
        if (qs != 0x100u) {
          const float S = __fmul_rn(scale_code_value(qs, args.scale_format), cs);
          nf4_decode64(c0, c1, S, o);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
      } else {
        const int j0 = (ks - main_steps) * 64;
        if (!B_MN) {  // fwd: B2 = lora B [N, r], row n0 + wr, cols j0..j0+63
          const int64_t n = n0 + wr;
          if (n < args.w_rows) {
            load_row128(args.lora_b2 + n * args.lora_ld + j0, args.lora_r - j0, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
        } else {      // dX: B2 = lora A [r, K], row j0 + wr, cols n0 + 64*fb ..
          const int jr = j0 + wr;
          const int64_t kf = n0 + 64 * fb;
          if (jr < args.lora_r && kf < args.w_cols) {
            load_row128(args.lora_b2 + (int64_t)jr * args.lora_ld + kf, 64, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
        }
      }
      if (!ptx::mbar_wait(&empty_b[sb], pb ^ 1, abort_flag)) return false;
      store_row128(sB + sb * C::B_STAGE + atom_off, row_in, o);
      // Each thread orders its own writes before the tensor core's reads and
      // arrives itself (one arrival per thread).
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&full_b[sb]);
      // refill this slot with the scale of the step two ahead; issued after the
      // arrive, whose release would otherwise wait for these loads
      scale_src(ptile, pks, qs, cs);
      advance(ptile, pks);
      if (++sb == C::SB) { sb = 0; pb ^= 1; }
      advance(tile, ks);
      return true;
    };
    while (ok && tile < num_tiles) {
      ok = produce(qa, ca);
      if (!ok || tile >= num_tiles) break;
      ok = produce(qb, cb);
    }
    if (!ok && lane == 0) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
