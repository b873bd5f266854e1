// Paged chunked prefill (placeholder until the tensor-core kernel lands).
#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

int launch_prefill(const PrefillArgs& a) {
  (void)a;
  return fail(PKV_ERR_UNSUPPORTED, "paged_attention_prefill: not built yet");
}

}  // namespace pkv
