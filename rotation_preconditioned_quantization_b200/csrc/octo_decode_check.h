// Host-side argument checks of the decode step, shared by octo_decode_attn
// and octo_decode_attn_static (internal to the library, not exported).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/octopus.h"

namespace octo {

// Every check of octo_decode_attn except the workspace pointer and size, in
// the same order and with the same status codes. On OCTO_OK, *ws_need holds
// the workspace bytes the call needs (octo_decode_attn_workspace). Touches
// no device state.
int decode_validate(const octo_layout* L, const octo_tables* tab, const void* q, int q_dtype, int B, int Hq, int Hkv,
                    int Lq, int64_t kv_len, int64_t cache_cap, const uint32_t* packed, const float* gamma,
                    const uint32_t* qjl_bits, const float* qjl_norm, const void* V, float scale, const float* out,
                    const float* logits, size_t* ws_need);

}  // namespace octo
