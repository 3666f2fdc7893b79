// One compiled variant of the scoring kernel (heads 32, head dim 128, BF16, pruning stage).
// Variants live in separate translation units so that they compile in parallel.
#include "score_topk.cuh"

namespace hwr {
void fill_variant_bf16_h32_d128_prune(ScoreVariant* v) { fill_variant<32, 128, false, true>(v); }
}  // namespace hwr
