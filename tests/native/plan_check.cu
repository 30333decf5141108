// Host-only driver for the decode kernel's shared-memory planner: prints one
// line per (G, max_gate_blocks, budget, kv dtype) with every region offset, for
// tests/test_plan.py to check alignment and overlap rules.
#include <cstdio>

#include "sas_internal.h"

int main() {
  const int mgs[] = {1, 63, 64, 512, 1023, 2048, 4096, 16384};
  const int budgets[] = {64, 1024, 2048, 4096, 16384};
  for (int G = 1; G <= sas::kMaxGroup; ++G)
    for (int mg : mgs)
      for (int b : budgets)
        for (int f32 = 0; f32 < 2; ++f32)
          for (int gated = 0; gated < 2; ++gated) {
            const sas::DecodeSmem p = sas::plan_decode_smem(G, mg, 8, 2, b / 64, f32 != 0, gated != 0);
            std::printf(
                "G=%d mg=%d budget=%d f32=%d gated=%d wq_heads=%d slots=%d sel=%d rows=%d gbias=%d qraw=%d qbar=%d pml=%d "
                "gam=%d bars=%d r_qv=%d r_wq=%d r_inbox=%d r_keys=%d r_hist=%d r_selbits=%d r_scan=%d "
                "r_lkeys=%d r_gather=%d total=%d ok=%d\n",
                G, mg, b, f32, gated, p.wq_heads, p.slots, p.sel, p.rows, p.gbias, p.qraw, p.qbar, p.pml, p.gam, p.bars, p.r_qv,
                p.r_wq, p.r_inbox, p.r_keys, p.r_hist, p.r_selbits, p.r_scan, p.r_lkeys, p.r_gather, p.total,
                sas::decode_smem_aligned(p, G, sas::kDim / 8) ? 1 : 0);
          }
  return 0;
}
