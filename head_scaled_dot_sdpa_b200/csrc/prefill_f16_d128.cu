// tcgen05 prefill kernel instances for __half, head_dim 128 (all bias / mask variants).
#include "prefill_sm100.cuh"

namespace sdpa {
namespace prefill {
SDPA_PREFILL_DEFINE_LAUNCH(__half, 128)
}  // namespace prefill
}  // namespace sdpa
