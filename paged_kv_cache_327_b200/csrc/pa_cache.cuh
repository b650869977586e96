// pa_cache.cuh -- the two cache kernels that feed decode attention.
//
// reshape_and_cache ("vLLM 深度解读", section 7): each new token's K and V rows (all KV
// heads of one token are contiguous, num_kv_heads * head_dim elements) go to their slot;
// in the [num_blocks, block_size, num_kv_heads, head_dim] cache, slot s is exactly row s
// of a [num_blocks * block_size, num_kv_heads * head_dim] view, so one token is one
// contiguous row copy.
// copy_blocks ("详解vLLM推理引擎架构", Copy-on-Write): one physical block is one contiguous
// block_bytes range of each cache.
// Both are plain 16-byte vector copies (bit-exact), bandwidth-bound, bounds-checked.
#pragma once

#include "pa_decode.cuh"

namespace pa {

__global__ void __launch_bounds__(128)
    pa_reshape_and_cache_kernel(const uint8_t* __restrict__ k, const uint8_t* __restrict__ v,
                                uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                const int64_t* __restrict__ slots, int num_tokens, int64_t row_bytes,
                                int64_t k_stride_bytes, int64_t v_stride_bytes, int64_t num_slots) {
  const int64_t vecs = row_bytes >> 4;
  for (int t = blockIdx.x; t < num_tokens; t += gridDim.x) {
    const int64_t s = slots[t];
    if (s < 0) continue;
    if (s >= num_slots) {
      if (threadIdx.x == 0) record_error(DEV_BAD_SLOT);
      continue;
    }
    const uint4* ks = reinterpret_cast<const uint4*>(k + t * k_stride_bytes);
    const uint4* vs = reinterpret_cast<const uint4*>(v + t * v_stride_bytes);
    uint4* kd = reinterpret_cast<uint4*>(kc + s * row_bytes);
    uint4* vd = reinterpret_cast<uint4*>(vc + s * row_bytes);
    for (int64_t i = threadIdx.x; i < vecs; i += blockDim.x) {
      const uint4 a = __ldg(ks + i), b = __ldg(vs + i);
      kd[i] = a;
      vd[i] = b;
    }
  }
}

// grid: (num_pairs, 2 [K, V], chunks)
__global__ void __launch_bounds__(256)
    pa_copy_blocks_kernel(uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                          const int32_t* __restrict__ pairs, int64_t num_blocks, int64_t block_bytes) {
  const int64_t src = pairs[2 * static_cast<int64_t>(blockIdx.x)];
  const int64_t dst = pairs[2 * static_cast<int64_t>(blockIdx.x) + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) record_error(DEV_BAD_PAIR);
    return;
  }
  uint8_t* base = blockIdx.y ? vc : kc;
  const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
  const int64_t vecs = block_bytes >> 4;
  for (int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.z) * blockDim.x; i < vecs;
       i += static_cast<int64_t>(blockDim.x) * gridDim.z)
    d[i] = s[i];
}

}  // namespace pa
