// Host-only driver: prints, for every GQA group size and list length the
// gate backward accepts, the K/V ring depth the library picks (as many
// stages, up to four, as fit in 227 KiB) and the kernel's dynamic shared
// memory, for tests/test_plan.py.
#include <cstdio>

#include "sas_internal.h"

int main() {
  for (int G = 1; G <= 8; ++G)
    for (int max_sel = 1; max_sel <= sas::kBwMaxSel; ++max_sel) {
      int stages = 4;
      while (stages > 1 && sas::gate_bwd_smem_bytes(G, max_sel, stages) > 227 * 1024) --stages;
      std::printf("G=%d max_sel=%d stages=%d bytes=%d\n", G, max_sel, stages,
                  sas::gate_bwd_smem_bytes(G, max_sel, stages));
    }
  return 0;
}
