// Library-internal entry points shared by the translation units of libattn.so (not exported).
#pragma once

#include "../../include/attn.h"

namespace attn {

// attn_prefill into a float32 partial: o [B, S, Hq, D] and lse [B, S, Hq] already hold the normalised
// output and log-sum-exp of the same rows over earlier key chunks, and this call merges its own
// result over keys [kv_pos0, kv_pos0 + T) into them by the exact log-sum-exp merge (rows that see
// none of these keys keep their stored values).  Used by the chunk streamer, which thus needs no
// per-task partial buffer and no separate merge pass.
attn_status_t prefill_accumulate_f32(const void* q, const void* k, const void* v, float* o, float* lse,
                                     attn_dims_t dims, int S, int T, int causal, long long q_pos0, long long kv_pos0,
                                     void* stream);

}  // namespace attn
