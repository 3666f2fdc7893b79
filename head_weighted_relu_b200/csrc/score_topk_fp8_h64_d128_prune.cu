// One compiled variant of the scoring kernel (heads 64, head dim 128, FP8 e4m3, pruning stage).
// Variants live in separate translation units so that they compile in parallel.
#include "score_topk.cuh"

namespace hwr {
void fill_variant_fp8_h64_d128_prune(ScoreVariant* v) { fill_variant<64, 128, true, true>(v); }
}  // namespace hwr
