// Host-only driver: prints the block-sparse prefill attention kernel's
// dynamic shared memory at every list length it accepts, for
// tests/test_plan.py to check that two CTAs still fit on one SM.
#include <cstdio>

#include "sas_prefill.cu"

int main() {
  for (int max_sel = 1; max_sel <= sas::kPfMaxSel; ++max_sel)
    std::printf("max_sel=%d bytes=%zu\n", max_sel, sas::prefill_attn_smem_bytes(max_sel));
  return 0;
}
