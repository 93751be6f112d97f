// tcgen05 prefill kernel instances for __nv_bfloat16, head_dim 128 (all bias / mask variants).
#include "prefill_sm100.cuh"

namespace sdpa {
namespace prefill {
SDPA_PREFILL_DEFINE_LAUNCH(__nv_bfloat16, 128)
}  // namespace prefill
}  // namespace sdpa
