// prefill.cu -- prefill path (rows above a few dozen).
#include "internal.h"

namespace moe {

size_t workspace_bytes(const moe_dims &d, int64_t rows) { return decode_layout(d, rows).total; }

bool prefill_available() { return false; }

int prefill_kernel_launches(const moe_dims &, int64_t) { return 0; }

int prefill_forward(const moe_dims &, const uint16_t *, int32_t, const uint16_t *, const uint8_t *,
                    const float *, const uint8_t *, const float *, const uint16_t *, uint16_t *,
                    const uint16_t *, const float *, void *, cudaStream_t, int32_t *, float *, float *)
{
    return MOE_EUNSUPPORTED;
}

}  // namespace moe
