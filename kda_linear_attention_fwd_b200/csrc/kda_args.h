// Host-side argument checks shared by the prefill entry points
// (kda_chunk_fwd / kda_chunk_fwd_ex and kda_chunk_fwd_noalloc), so that both
// accept and refuse exactly the same calls.  Each returns KDA_OK or the
// status the entry point must return; nothing is launched before they pass.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

inline bool is_aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
inline bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Sizes, head dimensions and element type.
inline int check_prefill_sizes(int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                               int32_t dv, kda_dtype dtype) {
    if (num_seqs < 0 || total_tokens < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// Buffers: required pointers, 16-byte alignment (plus `extra16`, e.g. the
// workspace, when not null), beta and cu_seqlens alignment, the only
// aliasing allowed (final_state == initial_state exactly), and the host copy
// of the offsets when given.  *empty is set when num_seqs == 0 and
// total_tokens == 0: a valid call with nothing to do.
inline int check_prefill_buffers(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const void *gate, const void *out,
                                 const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                 int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                                 int32_t dv, kda_dtype dtype, const float *initial_state,
                                 const float *final_state, const void *extra16, bool *empty) {
    *empty = false;
    if (num_seqs == 0) {
        if (total_tokens != 0) return KDA_ERR_INVALID_ARG;
        *empty = true;
        return KDA_OK;
    }
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const size_t esz = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const void *a16[] = {q, k, v, g, gate, out, initial_state, final_state, extra16};
    for (const void *p : a16)
        if (p && !is_aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    if (beta && !is_aligned(beta, esz)) return KDA_ERR_ALIGNMENT;
    if (!is_aligned(cu_seqlens, 4)) return KDA_ERR_ALIGNMENT;
    const size_t state_bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    if (initial_state && final_state && initial_state != final_state) {
        const char *a = (const char *)initial_state, *b = (const char *)final_state;
        if (a < b + state_bytes && b < a + state_bytes) return KDA_ERR_INVALID_ARG;
    }
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_tokens)
            return KDA_ERR_INVALID_ARG;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    }
    return KDA_OK;
}

// Status of a prefill from the first three words of its plan header (written
// on the device; read back after the stream has finished): [1] offsets
// inconsistent, [2] bit 4 = g out of range (checked build), bits 1 and 2 = a
// bounded device wait gave up.
inline int decode_plan_header(const int32_t h[3]) {
    if (h[1] != 0 || (h[2] & 4)) return KDA_ERR_INVALID_ARG;
    if (h[2] & 3) return KDA_ERR_TIMEOUT;
    return KDA_OK;
}

}  // namespace kda
