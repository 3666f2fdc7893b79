// Dispatch from (heads, head dim, FP8, pruning) to the compiled scoring-kernel variants.
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
void fill_variant_bf16_h32_d128_prune(ScoreVariant* v);
void fill_variant_bf16_h64_d128_prune(ScoreVariant* v);
void fill_variant_fp8_h32_d128_prune(ScoreVariant* v);
void fill_variant_fp8_h64_d128_prune(ScoreVariant* v);

bool score_variant(int H, int D, bool fp8, bool prune, ScoreVariant* v) {
  if (H == 4 && D == 64 && fp8 == false && prune == false) {
    fill_variant_bf16_h4_d64(v);
    return true;
  }
  if (H == 8 && D == 128 && fp8 == false && prune == false) {
    fill_variant_bf16_h8_d128(v);
    return true;
  }
  if (H == 16 && D == 64 && fp8 == false && prune == false) {
    fill_variant_bf16_h16_d64(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == false && prune == false) {
    fill_variant_bf16_h32_d128(v);
    return true;
  }
  if (H == 64 && D == 64 && fp8 == false && prune == false) {
    fill_variant_bf16_h64_d64(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == false && prune == false) {
    fill_variant_bf16_h64_d128(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == true && prune == false) {
    fill_variant_fp8_h32_d128(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == true && prune == false) {
    fill_variant_fp8_h64_d128(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == false && prune == true) {
    fill_variant_bf16_h32_d128_prune(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == false && prune == true) {
    fill_variant_bf16_h64_d128_prune(v);
    return true;
  }
  if (H == 32 && D == 128 && fp8 == true && prune == true) {
    fill_variant_fp8_h32_d128_prune(v);
    return true;
  }
  if (H == 64 && D == 128 && fp8 == true && prune == true) {
    fill_variant_fp8_h64_d128_prune(v);
    return true;
  }
  return false;
}

}  // namespace hwr
