// Host-side check of the decode GEMV's shared-memory placement: for every token
// count, K and stage count the launcher can choose, the buffers must fit the
// opt-in limit, keep their alignments and never overlap.  Built and run by
// tests/test_host_layout.py (host code only; no GPU needed).
#include <cstdio>
#include <vector>

#include "../../bit_nf4_quantized_27_b200/csrc/gemv_kernel.cuh"

using namespace qlora;

struct Region {
  uint32_t lo, hi;
  const char *what;
};

int main() {
  long checked = 0;
  int bad = 0;
  const uint32_t bases[] = {0u, 1024u};
  const int64_t ks[] = {256, 512, 768, 1024, 2048, 3072, 4096, 8192, 12288, 16384, 22016 / 64 * 64, 32768, 65536};
  for (uint32_t base : bases)
    for (int M = 1; M <= kGemvMaxM; ++M)
      for (int64_t K : ks) {
        if (!gemv_bulk_ok(16, K)) continue;
        const int64_t CH = K < 4096 ? K : 4096;
        for (int per = 1; per <= kBulkMaxRG; ++per) {
          const int uses = per * static_cast<int>(K / CH);
          const int S = gemv_bulk_stages(K, M, base, uses);
          if (S == 0) continue;
          ++checked;
          const uint32_t sb = gemv_bulk_stage_bytes(K), rb = gemv_bulk_red_bytes(M);
          const BulkLayout L = gemv_bulk_layout(base, sb, S, rb);
          const int bytes = gemv_bulk_smem_bytes(K, S, M, base);
          auto fail = [&](const char *why) {
            if (bad < 20) std::printf("M=%d K=%lld per=%d S=%d base=%u: %s\n", M, (long long)K, per, S, base, why);
            ++bad;
          };
          if (S < 2 || S > kBulkMaxStages) fail("stage count out of range");
          if (bytes > static_cast<int>(kBulkSmemLimit)) fail("exceeds the opt-in limit");
          if (L.end - base != static_cast<uint32_t>(bytes)) fail("end differs from the reported size");
          if (L.lut % 65536u) fail("table not 64 KB aligned");
          std::vector<Region> r;
          r.push_back({L.lut, L.lut + kBulkLutBytes, "table"});
          for (int i = 0; i < S; ++i) {
            if (L.stage[i] % 1024u) fail("stage not 1024-byte aligned");
            r.push_back({L.stage[i], L.stage[i] + sb, "stage"});
          }
          for (int i = 0; i < kBulkMaxRG; ++i) {
            if (L.red[i] % 16u) fail("partial sums not 16-byte aligned");
            r.push_back({L.red[i], L.red[i] + rb, "partial sums"});
          }
          if (L.bar % 8u) fail("barriers not 8-byte aligned");
          r.push_back({L.bar, L.bar + 2 * kBulkMaxStages * 8, "barriers"});
          for (const Region &a : r) {
            if (a.lo < base || a.hi > L.end) fail("region outside the window");
            for (const Region &b : r)
              if (&a < &b && a.lo < b.hi && b.lo < a.hi) fail("regions overlap");
          }
          // a stage must hold its codes and scale codes
          if (sb < 16 * CH / 2 + 16 * CH / 64) fail("stage too small");
        }
      }
  std::printf("checked %ld layouts, %d failures\n", checked, bad);
  return bad ? 1 : 0;
}
