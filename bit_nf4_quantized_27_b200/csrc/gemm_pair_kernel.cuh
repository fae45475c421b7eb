// The fused NF4 GEMM (forward and dX) on CTA pairs: a cluster of two CTAs on
// one TPC issues tcgen05 MMAs with cta_group::2, M = 256 (128 token rows in
// each CTA) and N = 256 (the decoded weight tile split 128 / 128 between the
// CTAs).  Against the single-CTA kernel this halves, per flop, the NF4 decoding
// each CTA does and the weight-operand bytes each CTA's tensor core reads from
// shared memory; each CTA still holds 2 x 128 x 256 fp32 accumulators (512
// TMEM columns) for the two 256-row halves of a 512 x 256 output tile.
//
//   D[M_rows, N_cols] = A . B^T (+ A2 . B2^T)     A, A2 by TMA; B, B2 decoded
//
// Roles per CTA (warp index): 0 TMA producer | 1 MMA issuer (even CTA only) +
// TMEM owner | 2..3 block scales | 4..7 epilogue | 8..15 NF4 decode, in two
// groups of 128 threads that take alternate K steps.  The block scales
// S = E4M3(q) * c2 reach the decode threads through a shared-memory ring, so the
// decode threads issue no global loads: their barrier arrivals (releases) then
// never wait on a load in flight.  Synchronisation across the pair:
//   * the even CTA's full_a / full_b barriers count both CTAs' A bytes (TMA
//     loads of either CTA complete on them) and both CTAs' decode arrivals;
//   * each MMA batch's commit arrives on empty_a / empty_b of both CTAs, the
//     last one of a tile on both CTAs' acc_full;
//   * both CTAs' epilogue warps arrive on the even CTA's acc_empty.
// Every mbarrier wait is bounded (a timeout raises QLORA_ERR_TIMEOUT and sets
// this CTA's abort flag); both CTAs meet at a cluster barrier before TMEM is
// freed and before either exits, so no CTA leaves while its peer may still
// touch its shared memory.
#pragma once

#include "gemm_kernel.cuh"

namespace qlora {

template <bool B_MN, int MT>
struct GemmPairCfg {
  static constexpr int BM = 128;                    // token rows per CTA per 256-row half tile
  static constexpr int BN = 256;                    // output columns per pair tile
  static constexpr int HB = 128;                    // weight-operand rows (N) per CTA
  static constexpr int BK = 64;
  static constexpr int A_STAGE = MT * BM * BK * 2;  // 32 KB at MT = 2
  static constexpr int B_STAGE = HB * BK * 2;       // 16 KB
  static constexpr int C_STAGE = HB * 32;           // codes: fwd 128 rows x 32 B, dX 64 rows x 64 B
  static constexpr int SA = 4, SB = 4, SC = 6;
  static constexpr int SS = 8;                      // block-scale ring (fp32 S per operand row)
  static constexpr int ACC_COLS = MT * BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 512;
  static constexpr int DEQ = 128;                   // decode threads per K step (one group)
  static constexpr int S_STAGE = HB * 4;
  static constexpr int SMEM_DATA = SA * A_STAGE + SB * B_STAGE + SC * C_STAGE + SS * S_STAGE;
  static constexpr int SMEM_BYTES = SMEM_DATA + 1024 /*align*/ + 512 /*barriers*/;
  static constexpr uint32_t IDESC = ptx::idesc_bf16(256, BN, 0, B_MN ? 1 : 0);
  static_assert(ACC_COLS <= TMEM_COLS, "TMEM");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <bool B_MN, int MT>
__global__ void __launch_bounds__(GemmPairCfg<B_MN, MT>::THREADS, 1)
gemm_nf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                     const __grid_constant__ CUtensorMap tmCodes, const GemmArgs args) {
  using C = GemmPairCfg<B_MN, MT>;
  extern __shared__ uint8_t smem_raw[];
  // Same offsets in both CTAs: the even CTA's descriptors address both.
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + C::SA * C::A_STAGE;
  uint8_t *sC = sB + C::SB * C::B_STAGE;
  float *sS = reinterpret_cast<float *>(sC + C::SC * C::C_STAGE);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sS + C::SS * C::HB);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + C::SA;
  uint64_t *full_b = empty_a + C::SA;
  uint64_t *empty_b = full_b + C::SB;
  uint64_t *full_c = empty_b + C::SB;
  uint64_t *empty_c = full_c + C::SC;
  uint64_t *full_s = empty_c + C::SC;
  uint64_t *empty_s = full_s + C::SS;
  uint64_t *acc_full = empty_s + C::SS;
  uint64_t *acc_empty = acc_full + 1;
  uint64_t *drain = acc_empty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the MMAs
  const bool even = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SA; ++s) { ptx::mbar_init(&full_a[s], 1); ptx::mbar_init(&empty_a[s], 1); }
    for (int s = 0; s < C::SB; ++s) { ptx::mbar_init(&full_b[s], 2 * C::DEQ); ptx::mbar_init(&empty_b[s], 1); }
    for (int s = 0; s < C::SC; ++s) { ptx::mbar_init(&full_c[s], 1); ptx::mbar_init(&empty_c[s], C::DEQ); }
    for (int s = 0; s < C::SS; ++s) { ptx::mbar_init(&full_s[s], 64); ptx::mbar_init(&empty_s[s], C::DEQ); }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 8);  // 4 epilogue warps in each CTA
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    if (args.lora_steps) ptx::prefetch_tmap(&tmA2);
    ptx::prefetch_tmap(&tmCodes);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA signal
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above overlaps the preceding kernel's tail; every global read and
  // write below comes after that kernel has completed.
  ptx::griddep_launch();
  ptx::griddep_wait();

  // Tiles of 2*128*MT tokens x 256 columns, handed out round-robin to the
  // clusters.  When the last round would leave at least half of the clusters
  // idle, its tiles are split into halves of 256 tokens (one accumulator), so
  // the last round takes half as long.
  const int num_m = (args.M_rows + 2 * C::BM * MT - 1) / (2 * C::BM * MT);
  const int num_n = (args.N_cols + C::BN - 1) / C::BN;
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const int full_tiles = num_m * num_n;
  const int rem = full_tiles % clusters;
  const bool split = MT == 2 && rem > 0 && 2 * rem <= clusters;
  const int main_tiles = split ? full_tiles - rem : full_tiles;
  const int num_tiles = split ? main_tiles + 2 * rem : full_tiles;
  auto tile_of = [&](int w, int &m0, int &n0, int &mt) {
    if (w < main_tiles) {
      m0 = (w % num_m) * 2 * C::BM * MT;
      n0 = (w / num_m) * C::BN;
      mt = MT;
    } else {
      const int f = main_tiles + ((w - main_tiles) >> 1);
      m0 = (f % num_m) * 2 * C::BM * MT + 2 * C::BM * ((w - main_tiles) & 1);
      n0 = (f / num_m) * C::BN;
      mt = 1;
    }
  };
  const int steps = args.k_steps + args.lora_steps;
  // operand row unit e (0..127) -> (W row offset wr, 64-feature block fb): fwd
  // W row nh + e; dX W row ks*64 + wr, features nh + 64 fb ..  (in every
  // quarter-warp of decode threads the code reads and the swizzled operand
  // writes fall on distinct banks)
  auto unit_map = [](int e, int &wr, int &fb) {
    if (!B_MN) {
      wr = e;
      fb = 0;
    } else {
      const int P = e >> 3, j = e & 7;
      wr = 8 * (P & 7) + j;
      fb = ((j >> 1) & 1) ^ (P >> 3);
    }
  };
  auto fail = [&]() {
    raise_status(args.status, QLORA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (ptx::elect_one()) {
      uint32_t sa = 0, pa = 0, sc = 0, pc = 0;
      int issued_a = 0, issued_c = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += clusters) {
        int m0, n0, mt;
        tile_of(tile, m0, n0, mt);
        const int nh = n0 + C::HB * static_cast<int>(rank);  // this CTA's first weight-operand row
        for (int ks = 0; ks < steps && ok; ++ks) {
          const bool lora = ks >= args.k_steps;
          if (!lora) {
            if (!ptx::mbar_wait(&empty_c[sc], pc ^ 1, abort_flag)) { ok = false; break; }
            ptx::mbar_arrive_expect_tx(&full_c[sc], C::C_STAGE);
            // fwd: W rows nh.., 32 code bytes of step ks; dX: 64 W rows, 64 code bytes from column nh
            if (!B_MN) ptx::tma_load_2d(sC + sc * C::C_STAGE, &tmCodes, &full_c[sc], ks * 32, nh);
            else ptx::tma_load_2d(sC + sc * C::C_STAGE, &tmCodes, &full_c[sc], nh / 2, ks * 64);
            ++issued_c;
            if (++sc == C::SC) { sc = 0; pc ^= 1; }
          }
          // empty_a is released by the even CTA's MMA commit, in both CTAs
          if (!ptx::mbar_wait(&empty_a[sa], pa ^ 1, abort_flag)) { ok = false; break; }
          if (even) ptx::mbar_arrive_expect_tx(&full_a[sa], 2 * mt * C::BM * C::BK * 2);
          const uint32_t bar = ptx::mapa_shared(ptx::smem_addr(&full_a[sa]), 0);
          uint8_t *dA = sA + sa * C::A_STAGE;
          for (int t = 0; t < mt; ++t) {
            const int row = m0 + t * 2 * C::BM + C::BM * static_cast<int>(rank);
            if (lora) ptx::tma_load_2d_pair(dA + t * 16384, &tmA2, bar, (ks - args.k_steps) * 64, row);
            else ptx::tma_load_2d_pair(dA + t * 16384, &tmA, bar, ks * 64, row);
          }
          ++issued_a;
          if (++sa == C::SA) { sa = 0; pa ^= 1; }
        }
      }
      if (!ok) fail();
      // Drain.  The even CTA's full_a completes only when both CTAs' copies have
      // landed; each CTA waits for its own code copies.
      if (even) {
        for (int i = 0; i < C::SA && i < issued_a; ++i) {
          if (sa == 0) { sa = C::SA - 1; pa ^= 1; } else { --sa; }
          ptx::mbar_wait(&full_a[sa], pa, nullptr);
        }
      }
      for (int i = 0; i < C::SC && i < issued_c; ++i) {
        if (sc == 0) { sc = C::SC - 1; pc ^= 1; } else { --sc; }
        ptx::mbar_wait(&full_c[sc], pc, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (even && ptx::elect_one()) {
      uint32_t sa = 0, pa = 0, sb = 0, pb = 0;
      int it = 0;
      bool ok = true;
      const uint32_t sA0 = ptx::smem_addr(sA), sB0 = ptx::smem_addr(sB);
      for (int tile = cluster; tile < num_tiles && ok; tile += clusters, ++it) {
        int m0_, n0_, mt;
        tile_of(tile, m0_, n0_, mt);
        if (!ptx::mbar_wait(acc_empty, (it & 1) ^ 1, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        for (int ks = 0; ks < steps && ok; ++ks) {
          if (!ptx::mbar_wait(&full_a[sa], pa, abort_flag)) { ok = false; break; }
          if (!ptx::mbar_wait(&full_b[sb], pb, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a_base = sA0 + sa * C::A_STAGE;
          const uint32_t b_base = sB0 + sb * C::B_STAGE;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_base + k16 * 2048, 8192, 1024)
                                     : ptx::smem_desc_sw128(b_base + k16 * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (t >= mt) break;
              const uint64_t ad = ptx::smem_desc_sw128(a_base + t * 16384 + k16 * 32, 16, 1024);
              ptx::mma_bf16_pair(tmem_base + t * C::BN, ad, bd, C::IDESC, (ks | k16) ? 1u : 0u);
            }
          }
          ptx::mma_commit_pair(&empty_a[sa], 0x3);
          ptx::mma_commit_pair(&empty_b[sb], 0x3);
          if (++sa == C::SA) { sa = 0; pa ^= 1; }
          if (++sb == C::SB) { sb = 0; pb ^= 1; }
        }
        if (ok) ptx::mma_commit_pair(acc_full, 0x3);
      }
      if (!ok) fail();
      // every pair MMA this thread issued has completed
      ptx::mma_commit_pair(drain, 0x1);
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp - 4;  // TMEM lane quadrant
    const uint32_t empty_even = ptx::mapa_shared(ptx::smem_addr(acc_empty), 0);
    int it = 0;
    for (int tile = cluster; tile < num_tiles; tile += clusters, ++it) {
      if (!ptx::mbar_wait(acc_full, it & 1, abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      ptx::tc_fence_after();
      int m0, n0, mt;
      tile_of(tile, m0, n0, mt);
      for (int t = 0; t < mt; ++t) {
        const int row = m0 + t * 2 * C::BM + C::BM * static_cast<int>(rank) + q * 32 + lane;
        for (int cb = 0; cb < C::BN; cb += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + t * C::BN + cb, v);
          ptx::tmem_ld_wait();
          const int col0 = n0 + cb;
          if (row < args.M_rows && col0 < args.N_cols) store_chunk32(args, row, col0, min(32, args.N_cols - col0), v);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_remote(empty_even);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ NF4 decode (both CTAs)
    const int d = threadIdx.x - 256;
    const int par = d >> 7;  // this group takes the flat K steps u with u % 2 == par
    const int e = d & 127;
    int wr, fb;
    unit_map(e, wr, fb);
    uint32_t atom_off, row_in, code_off, half_first;
    if (!B_MN) {
      atom_off = (e >> 3) * 1024;
      row_in = e & 7;
      code_off = e * 32;
      half_first = (e >> 2) & 1;
    } else {
      atom_off = fb * 8192 + (wr >> 3) * 1024;
      row_in = wr & 7;
      code_off = wr * 64 + fb * 32;
      half_first = ((e & 7) >> 2) & 1;
    }
    // flat step u -> (tile, ks) of this CTA's sequence
    int tile = cluster, ks = 0, u = par;
    auto advance = [&](int &t, int &k, int n) {
      for (int i = 0; i < n; ++i)
        if (++k == steps) { k = 0; t += clusters; }
    };
    advance(tile, ks, par);
    bool ok = true;
    auto produce = [&]() -> bool {
      const bool lora = ks >= args.k_steps;
      int m0_, n0, mt_;
      tile_of(tile, m0_, n0, mt_);
      const int nh = n0 + C::HB * static_cast<int>(rank);
      const uint32_t sb = static_cast<uint32_t>(u % C::SB), pb = static_cast<uint32_t>((u / C::SB) & 1);
      uint32_t o[32];
      if (!lora) {
        // the code stages advance once per non-LoRA step: index them by that count
        const int cu = (tile - cluster) / clusters * args.k_steps + ks;
        const uint32_t sc = static_cast<uint32_t>(cu % C::SC), pc = static_cast<uint32_t>((cu / C::SC) & 1);
        if (!ptx::mbar_wait(&full_c[sc], pc, abort_flag)) return false;
        const uint8_t *csrc = sC + sc * C::C_STAGE + code_off;
        const uint4 x0 = *reinterpret_cast<const uint4 *>(csrc + 16 * half_first);
        const uint4 x1 = *reinterpret_cast<const uint4 *>(csrc + 16 * (1 - half_first));
        ptx::mbar_arrive(&empty_c[sc]);
        const uint32_t ss = static_cast<uint32_t>(cu % C::SS), ps = static_cast<uint32_t>((cu / C::SS) & 1);
        if (!ptx::mbar_wait(&full_s[ss], ps, abort_flag)) return false;
        const float S = sS[ss * C::HB + e];
        ptx::mbar_arrive(&empty_s[ss]);
        const uint4 c0 = half_first ? x1 : x0, c1 = half_first ? x0 : x1;
        nf4_decode64(c0, c1, S, o);  // S = 0 past the weight's rows: the operand row is all (+-)0
      } else {
        const int j0 = (ks - args.k_steps) * 64;
        if (!B_MN) {  // fwd: B2 = LoRA B [N, r], row nh + wr, cols j0..j0+63
          const int64_t n = nh + wr;
          if (n < args.w_rows) {
            load_row128(args.lora_b2 + n * args.lora_ld + j0, args.lora_r - j0, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
        } else {      // dX: B2 = LoRA A [r, K], row j0 + wr, cols nh + 64 fb ..
          const int jr = j0 + wr;
          const int64_t kf = nh + 64 * fb;
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
      // each thread orders its own writes before the tensor core's reads and
      // arrives on the even CTA's barrier itself
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive_remote(ptx::mapa_shared(ptx::smem_addr(&full_b[sb]), 0));
      advance(tile, ks, 2);
      u += 2;
      return true;
    };
    while (ok && tile < num_tiles) ok = produce();
    if (!ok && lane == 0) fail();
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ block scales (both CTAs)
    // Thread t fills operand rows t and t + 64 of every non-LoRA step, loading
    // the scale codes and c2 of kNB steps at once so one load latency covers them.
    const int t = threadIdx.x - 64;
    const int64_t kblocks = args.w_cols / 64;
    int wr0, fb0, wr1, fb1;
    unit_map(t, wr0, fb0);
    unit_map(t + 64, wr1, fb1);
    constexpr int kNB = 4;
    int tile = cluster, ks = 0, cu = 0;
    bool ok = true;
    auto index_of = [&](int ti, int k, int wr, int fb) -> int64_t {  // flat block index, -1 = none
      int m0_, n0, mt_;
      tile_of(ti, m0_, n0, mt_);
      const int nh = n0 + C::HB * static_cast<int>(rank);
      int64_t wrow, kblk;
      if (!B_MN) { wrow = nh + wr; kblk = k; }
      else { wrow = (int64_t)k * 64 + wr; kblk = nh / 64 + fb; }
      return (wrow < args.w_rows && kblk < kblocks) ? wrow * kblocks + kblk : -1;
    };
    while (ok && tile < num_tiles) {
      uint32_t q[kNB][2];
      float c[kNB][2];
      int nb = 0, t2 = tile, k2 = ks;
#pragma unroll
      for (int b = 0; b < kNB; ++b) {
        q[b][0] = q[b][1] = 0u;
        c[b][0] = c[b][1] = 0.0f;
        if (t2 < num_tiles) {
          const int64_t i0 = index_of(t2, k2, wr0, fb0), i1 = index_of(t2, k2, wr1, fb1);
          if (i0 >= 0) { q[b][0] = __ldg(args.scale_codes + i0); c[b][0] = __ldg(args.c2 + (i0 >> 8)); }
          if (i1 >= 0) { q[b][1] = __ldg(args.scale_codes + i1); c[b][1] = __ldg(args.c2 + (i1 >> 8)); }
          ++nb;
          if (++k2 == args.k_steps) { k2 = 0; t2 += clusters; }
        }
      }
#pragma unroll
      for (int b = 0; b < kNB; ++b) {
        if (b < nb && ok) {
          const uint32_t ss = static_cast<uint32_t>((cu + b) % C::SS), ps = static_cast<uint32_t>(((cu + b) / C::SS) & 1);
          if (!ptx::mbar_wait(&empty_s[ss], ps ^ 1, abort_flag)) { ok = false; break; }
          sS[ss * C::HB + t] = __fmul_rn(scale_code_value(q[b][0], args.scale_format), c[b][0]);
          sS[ss * C::HB + t + 64] = __fmul_rn(scale_code_value(q[b][1], args.scale_format), c[b][1]);
          ptx::mbar_arrive(&full_s[ss]);
        }
      }
      cu += nb;
      tile = t2;
      ks = k2;
    }
    if (!ok && lane == 0) fail();
  }

  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
