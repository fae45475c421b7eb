// Host-side check of the quantiser's code search table: the table must pass its
// own self-checks (including the distance of every switch point from every cell
// edge), and this program prints the 15 switch points as float32 bit patterns so
// that tests/test_host_layout.py can compare them with the oracle's.  Host code
// only; no GPU needed.
#include <cstdio>

#include "../../bit_nf4_quantized_27_b200/csrc/host_common.h"

int main() {
  const qlora::HostCellTable &t = qlora::cell_table();
  std::printf("ok %d\n", t.ok ? 1 : 0);
  std::printf("min_edge_ulps %u\n", t.min_edge_ulps);
  for (int j = 0; j < 15; ++j) std::printf("switch %d %08x\n", j, qlora::f32_bits(t.switch_points[j]));
  return t.ok ? 0 : 1;
}
