// One compiled variant of the scoring kernel (heads 4, head dim 64, BF16).
// Variants live in separate translation units so that they compile in parallel.
#include "score_topk.cuh"

namespace hwr {
void fill_variant_bf16_h4_d64(ScoreVariant* v) { fill_variant<4, 64, false, false>(v); }
}  // namespace hwr
