// KV append: PagedKVCache's logical-to-physical write (BareLLM README,
// component list).  Request i's new token, all KV heads, is one contiguous
// run of Hkv*D elements in both k_new and the NHD pool, so the kernel is a
// 16-byte vector scatter: thread j of the flattened (request, vector) range
// copies one vector of K and one of V.  Slots < 0 are skipped; slots past the
// pool are skipped and recorded in the error word (no trap).
#pragma once

#include "common.cuh"

namespace pa {

__global__ void __launch_bounds__(256) kv_append_kernel(const uint4 *__restrict__ k_new,
                                                        const uint4 *__restrict__ v_new,
                                                        const int32_t *__restrict__ slot_mapping,
                                                        uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                                        int32_t B, int32_t vec_per_token, int64_t num_slots,
                                                        int32_t *error) {
    // a decode grid launched after this one may run its prologue meanwhile; it
    // waits for this grid's completion before reading any K/V row
    grid_launch_dependents();
    const int64_t total = (int64_t)B * vec_per_token;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t b = (int32_t)(i / vec_per_token);
        const int32_t v = (int32_t)(i - (int64_t)b * vec_per_token);
        const int32_t slot = __ldg(slot_mapping + b);
        if (slot < 0) continue;
        if ((int64_t)slot >= num_slots) {
            if (v == 0) set_error(error, PA_DEVERR_SLOT);
            continue;
        }
        const int64_t dst = (int64_t)slot * vec_per_token + v;
        const uint4 kv = __ldg(k_new + i);
        const uint4 vv = __ldg(v_new + i);
        k_cache[dst] = kv;
        v_cache[dst] = vv;
    }
}

}  // namespace pa
