// One compiled variant of the scoring kernel (heads 32, head dim 128, BF16).
// Variants live in separate translation units so that they compile in parallel.
#include "score_topk.cuh"

namespace hwr {
void fill_variant_bf16_h32_d128(ScoreVariant* v) { fill_variant<32, 128, false, false>(v); }
}  // namespace hwr
