// Dispatch from (heads, head dim, FP8) to the compiled scoring-kernel variants.
#include "internal.h"

namespace hwr {

void fill_variant_bf16_h4_d64(ScoreVariant* v);
void fill_variant_bf16_h8_d128(ScoreVariant* v);
void fill_variant_bf16_h16_d64(ScoreVariant* v);
void fill_variant_bf16_h32_d128(ScoreVariant* v);
void fill_variant_bf16_h64_d64(ScoreVariant* v);
void fill_variant_bf16_h64_d128(ScoreVariant* v);
void fill_variant_fp8_h32_d128(ScoreVariant* v);
void fill_variant_fp8_h64_d128(ScoreVariant* v);

bool score_variant(int H, int D, bool fp8, ScoreVariant* v) {
  if (H == 4 && D == 64 && fp8 == false) {
    fill_variant_bf16_h4_d64(v);
    return true;
  }
  if (H == 8 && D == 128 && fp8 == false) {
    fill_variant_bf16_h8_d128(v);
    return true;
  }
  if (H == 16 && D == 64 && fp8 == false) {
    fill_variant_bf16_h16_d64(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == false) {
    fill_variant_bf16_h32_d128(v);
    return true;
  }
  if (H == 64 && D == 64 && fp8 == false) {
    fill_variant_bf16_h64_d64(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == false) {
    fill_variant_bf16_h64_d128(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == true) {
    fill_variant_fp8_h32_d128(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == true) {
    fill_variant_fp8_h64_d128(v);
    return true;
  }
  return false;
}

}  // namespace hwr
