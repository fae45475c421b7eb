// Host-side check of the one-kernel decode path's plan: for every shape, token
// count, rank, SM count and window start the launcher can see, the shared-memory
// buffers must fit the opt-in limit, keep their alignments (copy destinations on
// 16 bytes, the swizzled ring and B rows on 1024, the pair table on 64 KB) and
// never overlap; the CTAs' unit ranges
// must cover every row exactly once; and the per-CTA buffers must hold the
// largest CTA's units.  Built and run by tests/test_host_layout.py (host code
// only; no GPU needed).
#include <algorithm>
#include <cstdio>
#include <vector>

#include "../../bit_nf4_quantized_27_b200/csrc/decode_kernel.cuh"

using namespace qlora;

struct Region {
  uint32_t lo, hi;
};

int main() {
  long checked = 0;
  int bad = 0;
  const uint32_t bases[] = {0u, 1024u};
  const int64_t ks[] = {256, 512, 768, 1024, 1280, 2048, 3072, 3840, 4096};
  const int64_t ns[] = {8, 16, 24, 256, 328, 1040, 2064, 4096, 4816, 11008, 22016, 32768, 65536};
  const int rs[] = {8, 16, 24, 48, 64, 96, 128, 192, 256};
  const int smss[] = {148, 132, 8, 1};
  for (uint32_t base : bases)
    for (int sms : smss)
      for (int64_t K : ks)
        for (int64_t N : ns)
          for (int r : rs)
            for (int M = 1; M <= kGemvMaxM; ++M) {
              const DecodePlan p = decode_plan(N, K, M, r, sms, base);
              auto fail = [&](const char *why) {
                if (bad < 20)
                  std::printf("N=%lld K=%lld M=%d r=%d sms=%d base=%u: %s\n", (long long)N, (long long)K, M, r, sms,
                              base, why);
                ++bad;
              };
              if (!decode_shape_ok(K, r)) {
                if (p.ok) fail("plan for an unsupported shape");
                continue;
              }
              if (!p.ok) {
                // the launcher then takes the two-kernel path; that is allowed only for
                // ranks above 64 (the CTA's B rows take r * 2 bytes per row), very
                // tall weights (many units per CTA) or a GPU far smaller than a
                // B200 (which puts more units on a CTA)
                if (N <= 16384 && r <= 64 && sms >= 132) fail("no plan for a supported shape");
                continue;
              }
              ++checked;
              const DecodeLayout &L = p.lay;
              const int rows_per_unit = 16 * p.RPS;
              if (p.WPR * p.RPS > kDecWarps || p.WPR * 256 != K) fail("warp split");
              if ((int64_t)p.units * rows_per_unit < N || (int64_t)(p.units - 1) * rows_per_unit >= N)
                fail("units do not cover the rows exactly");
              if (p.G < 1 || p.G > sms || p.G > p.units) fail("grid size");
              int most = 0, covered = 0;
              for (int c = 0; c < p.G; ++c) {
                // the kernel's split: the first units % G CTAs take one unit more
                const int per = p.units / p.G, extra = p.units % p.G;
                const int u0 = c * per + (c < extra ? c : extra), u1 = u0 + per + (c < extra ? 1 : 0);
                if (u0 != covered) fail("unit ranges not contiguous");
                covered = u1;
                if (u1 - u0 < 1) fail("a CTA without units");
                most = most > u1 - u0 ? most : u1 - u0;
              }
              if (covered != p.units) fail("unit ranges do not end at the last unit");
              if (most > p.units_max) fail("units_max below the largest CTA");
              if (p.stages < 2 || p.stages > kDecMaxStages) fail("stage count");
              if (p.F < 1 || p.F > p.units_max) fail("round size");
              if (p.dyn_bytes > (int)kDecSmemLimit || L.end - base != (uint32_t)p.dyn_bytes) fail("window size");
              if (L.lut % 65536u || L.lut < base) fail("table alignment");
              const int64_t crows = (int64_t)p.units_max * rows_per_unit;  // rows of the largest CTA
              if (p.ring_bytes != (uint32_t)(p.stages * kDecWarps * kDecWarpStage)) fail("ring bytes");
              // decoded scales: 16-byte aligned rows, and the eight rows a warp reads
              // at once (16 bytes each) start in eight different bank quads
              const int sfs = decode_sf_stride((int)(K / 64));
              if (sfs < K / 64 || sfs % 4 != 0) fail("scale table stride");
              bool quads[8] = {};
              for (int rr = 0; rr < 8; ++rr) quads[((rr * sfs) % 32) / 4] = true;
              for (bool b : quads)
                if (!b) fail("scale table bank conflict");
              if (p.sf_bytes != (uint32_t)(crows * sfs * 4)) fail("scale table bytes");
              const int chunks = (r + 63) / 64;
              if (p.chunks != chunks || p.brow_unit_bytes != (uint32_t)(chunks * rows_per_unit * 128) ||
                  p.brows_bytes != p.units_max * p.brow_unit_bytes || p.brow_unit_bytes % 1024u)
                fail("B row bytes");
              if (p.stf_bytes != (uint32_t)(((r + 15) / 16) * p.NG * 32 * 4 * 8)) fail("entry bytes");
              if (p.stf_bytes > (uint32_t)(((r + 15) / 16) * 2048)) fail("entries exceed the workspace share");
              if (p.yacc_bytes != (uint32_t)(crows * p.TR * 4)) fail("sum bytes");
              std::vector<Region> reg;
              reg.push_back({L.lut, L.lut + kDecLutBytes});
              if (L.ring % 1024u) fail("ring alignment");
              reg.push_back({L.ring, L.ring + p.ring_bytes});
              if (L.sf % 16u) fail("scale table alignment");
              reg.push_back({L.sf, L.sf + p.sf_bytes});
              if (L.brows % 1024u) fail("B rows alignment");
              reg.push_back({L.brows, L.brows + p.brows_bytes});
              if (p.red_unit_bytes != (uint32_t)(kDecWarps * 17 * p.TR * 4)) fail("partial slot bytes");
              if (L.red % 16u) fail("red alignment");
              reg.push_back({L.red, L.red + (uint32_t)p.F * p.red_unit_bytes});
              if (L.yacc % 16u) fail("sum alignment");
              reg.push_back({L.yacc, L.yacc + p.yacc_bytes});
              if (L.stf % 16u) fail("entry alignment");
              reg.push_back({L.stf, L.stf + p.stf_bytes});
              if (L.bar % 8u) fail("barrier alignment");
              reg.push_back({L.bar, L.bar + kDecBarBytes});
              reg.push_back({L.misc, L.misc + 32});
              for (size_t x = 0; x < reg.size(); ++x) {
                if (reg[x].lo < base || reg[x].hi > L.end) fail("region outside the window");
                for (size_t y = x + 1; y < reg.size(); ++y)
                  if (reg[x].lo < reg[y].hi && reg[y].lo < reg[x].hi) fail("overlapping regions");
              }
            }
  std::printf("%ld plans checked, %d failures\n", checked, bad);
  return bad ? 1 : 0;
}
