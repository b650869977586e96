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
  // two tokens per iteration (t and t + gridDim.x): their rows are read together with their slots
  // (the loads do not wait for each other); a slot only decides whether, and where, a row is stored
  for (int t = blockIdx.x; t < num_tokens; t += 2 * gridDim.x) {
    const int t2 = t + gridDim.x;
    const bool two = t2 < num_tokens;
    const int64_t s = slots[t], s2 = two ? slots[t2] : -1;
    const bool st = s >= 0 && s < num_slots, st2 = s2 >= 0 && s2 < num_slots;
    if (threadIdx.x == 0 && (s >= num_slots || s2 >= num_slots)) record_error(DEV_BAD_SLOT);
    const uint4* ks = reinterpret_cast<const uint4*>(k + t * k_stride_bytes);
    const uint4* vs = reinterpret_cast<const uint4*>(v + t * v_stride_bytes);
    const uint4* ks2 = reinterpret_cast<const uint4*>(k + (two ? t2 : t) * k_stride_bytes);
    const uint4* vs2 = reinterpret_cast<const uint4*>(v + (two ? t2 : t) * v_stride_bytes);
    uint4* kd = reinterpret_cast<uint4*>(kc + (st ? s : 0) * row_bytes);
    uint4* vd = reinterpret_cast<uint4*>(vc + (st ? s : 0) * row_bytes);
    uint4* kd2 = reinterpret_cast<uint4*>(kc + (st2 ? s2 : 0) * row_bytes);
    uint4* vd2 = reinterpret_cast<uint4*>(vc + (st2 ? s2 : 0) * row_bytes);
    for (int64_t i = threadIdx.x; i < vecs; i += blockDim.x) {
      const uint4 a = __ldg(ks + i), b = __ldg(vs + i);
      uint4 a2 = a, b2 = b;
      if (two) {
        a2 = __ldg(ks2 + i);
        b2 = __ldg(vs2 + i);
      }
      if (st) {
        kd[i] = a;
        vd[i] = b;
      }
      if (st2) {
        kd2[i] = a2;
        vd2[i] = b2;
      }
    }
  }
}

// Store into an FP8 E4M3 cache: each element x of the token's K (V) row becomes the code
// e4m3(x / scale), the division rounded to nearest in fp32, the conversion rounded to
// nearest even and saturated to +-448.  A thread converts 8 consecutive elements.
template <typename IT>
__device__ __forceinline__ void load8(const IT* p, float (&x)[8]) {
  if constexpr (std::is_same<IT, float>::value) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
  } else {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const IT* e = reinterpret_cast<const IT*>(&u);
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = to_float(e[j]);
  }
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);  // a: low byte
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xffffu) | (hi << 16);
}

template <typename IT>
__global__ void __launch_bounds__(128)
    pa_reshape_and_cache_fp8_kernel(const IT* __restrict__ k, const IT* __restrict__ v,
                                    uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                    const int64_t* __restrict__ slots, int num_tokens, int64_t row,
                                    int64_t k_stride, int64_t v_stride, int64_t num_slots, float k_scale,
                                    float v_scale) {
  for (int t = blockIdx.x; t < num_tokens; t += gridDim.x) {
    // as in the 16-bit store, the rows are read together with the slot, which only guards the stores
    const int64_t s = slots[t];
    const bool store = s >= 0 && s < num_slots;
    if (s >= num_slots && threadIdx.x == 0) record_error(DEV_BAD_SLOT);
    for (int64_t i = threadIdx.x * 8; i < row; i += blockDim.x * 8) {
      float x[2][8];
      load8(k + t * k_stride + i, x[0]);
      load8(v + t * v_stride + i, x[1]);
      if (!store) continue;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float sc = which ? v_scale : k_scale;
#pragma unroll
        for (int j = 0; j < 8; ++j) x[which][j] = __fdiv_rn(x[which][j], sc);
        const uint2 w = make_uint2(e4m3x4(x[which][0], x[which][1], x[which][2], x[which][3]),
                                   e4m3x4(x[which][4], x[which][5], x[which][6], x[which][7]));
        *reinterpret_cast<uint2*>((which ? vc : kc) + s * row + i) = w;
      }
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
  const int64_t stride = static_cast<int64_t>(blockDim.x) * gridDim.z;
  int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.z) * blockDim.x;
  for (; i + 3 * stride < vecs; i += 4 * stride) {  // four 16-byte loads in flight per thread
    const uint4 a = s[i], b = s[i + stride], c = s[i + 2 * stride], e = s[i + 3 * stride];
    d[i] = a;
    d[i + stride] = b;
    d[i + 2 * stride] = c;
    d[i + 3 * stride] = e;
  }
  for (; i < vecs; i += stride) d[i] = s[i];
}

}  // namespace pa

namespace pa {

// Swap: block pairs[p][0] of the source pool goes to block pairs[p][1] of the destination pool
// (K and V).  Either pool may be pinned host memory the device addresses directly, so each
// thread keeps four independent 16-byte loads in flight to cover the host link's latency.
// grid: (num_pairs, 2 [K, V], chunks)
__global__ void __launch_bounds__(256)
    pa_swap_blocks_kernel(uint8_t* __restrict__ dk, uint8_t* __restrict__ dv, const uint8_t* __restrict__ sk,
                          const uint8_t* __restrict__ sv, const int32_t* __restrict__ pairs, int64_t num_src,
                          int64_t num_dst, int64_t block_bytes) {
  const int64_t src = pairs[2 * static_cast<int64_t>(blockIdx.x)];
  const int64_t dst = pairs[2 * static_cast<int64_t>(blockIdx.x) + 1];
  if (src < 0 || src >= num_src || dst < 0 || dst >= num_dst) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) record_error(DEV_BAD_PAIR);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>((blockIdx.y ? sv : sk) + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>((blockIdx.y ? dv : dk) + dst * block_bytes);
  const int64_t vecs = block_bytes >> 4;
  const int64_t stride = static_cast<int64_t>(blockDim.x) * gridDim.z;
  int64_t i = threadIdx.x + static_cast<int64_t>(blockIdx.z) * blockDim.x;
  for (; i + 3 * stride < vecs; i += 4 * stride) {
    const uint4 a = s[i], b = s[i + stride], c = s[i + 2 * stride], e = s[i + 3 * stride];
    d[i] = a;
    d[i + stride] = b;
    d[i + 2 * stride] = c;
    d[i + 3 * stride] = e;
  }
  for (; i < vecs; i += stride) d[i] = s[i];
}

}  // namespace pa
