// pa_decode.cuh -- split-K paged decode attention for sm_100a.
//
// What is computed ("vLLM 深度解读", section 3, PagedAttention CUDA kernel): for each
// sequence i and query head hq, softmax over the sequence's tokens of
// scale * q[i,hq,:] . K_t, applied to V_t, where token t of sequence i sits in physical
// block block_tables[i][t / block_size] at position t % block_size, KV head hq / G.
//
// How (B200 design, not the page's one-CTA-per-(seq, head) scalar loop):
//  * plan kernel: one CTA turns seq_lens into a work list of (sequence, partition)
//    pairs -- full 512-token partitions first, the ragged tails last -- and zeroes the
//    work counter;
//  * partition kernel: persistent, one CTA per SM, each warp an independent worker.  A
//    work item is (sequence, partition, KV head).  The warp grabs items with an atomic
//    counter and streams the item's pages through its own ring of shared-memory slots:
//    lane 0 issues one TMA per 64-column half of the K and V page (box = block_size
//    rows x 128 B, 128-byte swizzle, L2 evict-first) plus a bulk copy of the G query
//    rows with the first page, all counted on the slot's mbarrier.  The ring runs
//    across item boundaries, so the warp keeps NSLOT pages in flight at all times.
//    Per page the G grouped query heads share one read of K and V:
//      S^T[tokens x G] = K[tokens x D] . Q^T[D x G]        (mma.sync m16n8k16, fp32 acc)
//      online softmax per query head (exp2 on scale*log2(e)-scaled scores)
//      O^T[D x G]    += V^T[D x tokens] . P^T[tokens x G]  (P^T via movmatrix.trans)
//    A sequence that fits one partition writes `out` directly; longer ones write the
//    partition's (max, sum, unnormalised O) to the workspace;
//  * reduce kernel: merges a sequence's partitions with the log-sum-exp rescale.
// The partition boundaries depend only on seq_lens[i], and each item is computed the
// same way whatever warp runs it, so results are deterministic and batch-invariant.
#pragma once

#include <math_constants.h>

#include "pa_ptx.cuh"

namespace pa {

enum : unsigned {
  DEV_OK = 0,
  DEV_BAD_BLOCK_ID = 1,
  DEV_BAD_SEQ_LEN = 2,
  DEV_BAD_SLOT = 3,
  DEV_BAD_PAIR = 4,
  DEV_TIMEOUT = 5,
};

enum : int { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

// First data-dependent fault seen by any kernel of this library on this device.
__device__ unsigned int g_dev_error;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_dev_error, 0u, code); }

// polls of an mbarrier before a wait is declared dead
constexpr uint32_t kWaitLimit = 1u << 20;

struct WorkItem {
  int seq, part, len, pad;
};

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int num_seqs, num_q_heads, num_kv_heads, group;
  int head_dim, block_size, max_blocks_per_seq, num_blocks;
  int partition_size, max_parts, out_dtype, pad;
  float scale_log2;  // scale * log2(e)
  // workspace views
  unsigned int* counters;  // [0] next work item, [1] number of (sequence, partition) pairs
  int* seq_nparts;         // [num_seqs]: partitions of the sequence, 0 if empty, -1 if invalid
  WorkItem* items;         // [num_seqs * max_parts]
  float2* part_ml;         // [num_seqs * max_parts * num_q_heads]: (max in log2 units, sum)
  float* part_acc;         // [num_seqs * max_parts * num_q_heads * head_dim]
};

__device__ __forceinline__ void store_out(void* out, int64_t idx, float v, int dt) {
  if (dt == DT_F32)
    static_cast<float*>(out)[idx] = v;
  else if (dt == DT_BF16)
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  else
    static_cast<__half*>(out)[idx] = __float2half_rn(v);
}

// ------------------------------------------------------------------------------ plan
__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive prefix sum over a 1024-thread block; *total receives the block sum.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int inc = warp_inclusive_scan(v);
  if (lane == 31) s_warp[w] = inc;
  __syncthreads();
  if (w == 0) {
    const int x = s_warp[lane];
    const int xi = warp_inclusive_scan(x);
    s_warp[lane] = xi - x;
    if (lane == 31) s_warp[32] = xi;
  }
  __syncthreads();
  const int r = s_warp[w] + inc - v;
  *total = s_warp[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) pa_decode_plan_kernel(const DecodeParams p) {
  __shared__ int s_warp[33];
  const int N = p.num_seqs, P = p.partition_size;
  const int max_len = p.max_blocks_per_seq * p.block_size;
  int local = 0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int L = p.seq_lens[i];
    if (L >= 0 && L <= max_len) local += L / P;
  }
  int n_full;
  block_exclusive_scan(local, s_warp, &n_full);
  int base_full = 0, base_tail = 0;
  for (int start = 0; start < N; start += blockDim.x) {
    const int i = start + threadIdx.x;
    int L = 0, nf = 0, nt = 0;
    if (i < N) {
      L = p.seq_lens[i];
      const bool valid = L >= 0 && L <= max_len;
      if (valid) {
        nf = L / P;
        nt = (L % P) ? 1 : 0;
      } else {
        record_error(DEV_BAD_SEQ_LEN);
      }
      p.seq_nparts[i] = valid ? nf + nt : -1;
    }
    int tf, tt;
    const int of = block_exclusive_scan(nf, s_warp, &tf);
    const int ot = block_exclusive_scan(nt, s_warp, &tt);
    for (int k = 0; k < nf; ++k) p.items[base_full + of + k] = WorkItem{i, k, L, 0};
    if (nt) p.items[n_full + base_tail + ot] = WorkItem{i, nf, L, 0};
    base_full += tf;
    base_tail += tt;
  }
  if (threadIdx.x == 0) {
    p.counters[0] = 0;
    p.counters[1] = static_cast<unsigned>(n_full + base_tail);
  }
}

// ------------------------------------------------------------------------------ partition kernel
template <int BS, int D, typename KT, bool QF32>
struct DecodeCfg {
  static constexpr int HALVES = D / 64;                 // 64-element (128-byte) column halves
  static constexpr int BOX_BYTES = BS * 128;            // one TMA box: BS rows x 128 bytes
  static constexpr int PAGE_BYTES = BOX_BYTES * HALVES; // one KV head of one block
  static constexpr int QE = QF32 ? 4 : 2;
  static constexpr int Q_BYTES = 8 * D * QE;            // up to 8 grouped query rows
  static constexpr int SLOT_BYTES = ((2 * PAGE_BYTES + Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int NWARP = 4;
  static constexpr int SMEM_BUDGET = 200 * 1024;
  static constexpr int NSLOT_FIT = SMEM_BUDGET / (NWARP * SLOT_BYTES);
  static constexpr int NSLOT = NSLOT_FIT > 8 ? 8 : (NSLOT_FIT < 2 ? 2 : NSLOT_FIT);
  static constexpr int RING_BYTES = NWARP * NSLOT * SLOT_BYTES;
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + NWARP * NSLOT * (8 + 16);
  static constexpr int MT = BS / 16;    // 16-token MMA tiles per page
  static constexpr int KS = D / 16;     // 16-wide steps over head_dim
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(BS == 16 || BS == 32, "block_size");
};

// byte offset, inside a page, of the 16-byte chunk holding (row t, columns d0..d0+7)
// under the TMA 128-byte swizzle (chunk index XOR row mod 8 within each 1024-byte atom)
template <int BOX_BYTES>
__device__ __forceinline__ uint32_t swz(int t, int d0) {
  return (d0 >> 6) * BOX_BYTES + t * 128 + ((((d0 & 63) >> 3) ^ (t & 7)) << 4);
}

template <int BS, int D, typename KT, bool QF32>
__global__ void __launch_bounds__(DecodeCfg<BS, D, KT, QF32>::NWARP * 32, 1)
    pa_decode_partition_kernel(const __grid_constant__ CUtensorMap tmk,
                               const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
  using C = DecodeCfg<BS, D, KT, QF32>;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int F_FIRST = 1, F_LAST = 2, F_BAD = 4, F_SINGLE = 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * C::NSLOT * C::SLOT_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES) + warp * C::NSLOT;
  int4* meta = reinterpret_cast<int4*>(smem + C::RING_BYTES + C::NWARP * C::NSLOT * 8) + warp * C::NSLOT;

  // query rows >= G of every slot stay zero: the bulk copy only ever writes rows < G
  for (int s = 0; s < C::NSLOT; ++s) {
    uint4* qz = reinterpret_cast<uint4*>(ring + s * C::SLOT_BYTES + 2 * C::PAGE_BYTES);
    for (int i = lane; i < C::Q_BYTES / 16; i += 32) qz[i] = make_uint4(0, 0, 0, 0);
  }
  if (lane == 0) {
    for (int s = 0; s < C::NSLOT; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    if (warp == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
  }
  __syncwarp();

  const int G = p.group, Hkv = p.num_kv_heads, Hq = p.num_q_heads;
  const unsigned total = p.counters[1] * static_cast<unsigned>(Hkv);
  const uint64_t pol = policy_evict_first();

  // ---------------- producer state (warp-uniform, except f_bt: lane i holds page i's block id)
  int f_seq = 0, f_part = 0, f_kvh = 0, f_tok0 = 0, f_tok1 = 0, f_len = 0, f_npages = 0, f_page = 0;
  int f_bt = 0;
  bool f_bad = false, f_done = false;
  uint32_t n_fetch = 0, n_cons = 0;

  auto next_item = [&]() -> bool {
    unsigned w = 0;
    if (lane == 0) w = atomicAdd(&p.counters[0], 1u);
    w = __shfl_sync(FULL, w, 0);
    if (w >= total) return false;
    const WorkItem it = p.items[w / Hkv];
    f_kvh = static_cast<int>(w % Hkv);
    f_seq = it.seq;
    f_part = it.part;
    f_len = it.len;
    f_tok0 = f_part * p.partition_size;
    f_tok1 = min(f_len, f_tok0 + p.partition_size);
    f_npages = (f_tok1 - f_tok0 + BS - 1) / BS;
    f_page = 0;
    bool bad = false;
    f_bt = 0;
    if (lane < f_npages) {
      f_bt = p.block_tables[static_cast<int64_t>(f_seq) * p.max_blocks_per_seq + f_tok0 / BS + lane];
      bad = f_bt < 0 || f_bt >= p.num_blocks;
    }
    f_bad = __any_sync(FULL, bad);
    if (f_bad && lane == 0) record_error(DEV_BAD_BLOCK_ID);
    return true;
  };

  // Issue the loads of the next page into slot n_fetch % NSLOT (whose previous page has
  // been consumed).  Returns false once the work list is exhausted.
  auto fetch = [&]() -> bool {
    if (f_done) return false;
    if (f_page >= f_npages && !next_item()) {
      f_done = true;
      return false;
    }
    const int phys = __shfl_sync(FULL, f_bt, f_page);
    const int slot = static_cast<int>(n_fetch % C::NSLOT);
    if (lane == 0) {
      uint8_t* sb = ring + slot * C::SLOT_BYTES;
      const int ntok = min(BS, f_tok1 - (f_tok0 + f_page * BS));
      const int flags = (f_page == 0 ? F_FIRST : 0) | (f_page == f_npages - 1 ? F_LAST : 0) |
                        (f_bad ? F_BAD : 0) | (f_len <= p.partition_size ? F_SINGLE : 0);
      meta[slot] = make_int4(f_seq, f_part, f_kvh, (ntok << 8) | flags);
      if (f_bad) {
        mbar_arrive(&bars[slot]);
      } else {
        const uint32_t qbytes = f_page == 0 ? static_cast<uint32_t>(G * D * C::QE) : 0u;
        mbar_arrive_expect_tx(&bars[slot], 2 * C::PAGE_BYTES + qbytes);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h) {
          tma_load_3d(sb + h * C::BOX_BYTES, &tmk, 0, f_kvh * C::HALVES + h, phys * BS, &bars[slot], pol);
          tma_load_3d(sb + C::PAGE_BYTES + h * C::BOX_BYTES, &tmv, 0, f_kvh * C::HALVES + h, phys * BS,
                      &bars[slot], pol);
        }
        if (qbytes)
          bulk_load(sb + 2 * C::PAGE_BYTES,
                    static_cast<const uint8_t*>(p.q) +
                        (static_cast<int64_t>(f_seq) * Hq + f_kvh * G) * D * C::QE,
                    qbytes, &bars[slot]);
      }
    }
    ++f_page;
    ++n_fetch;
    return true;
  };

  // ---------------- consumer state
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};
  float acc[C::KS][4];
  uint32_t qf[C::KS][2];
  uint32_t ql[QF32 ? C::KS : 1][2];
  bool poisoned = false;
  const int lr = lane & 7, lm = lane >> 3;  // ldmatrix: row inside an 8x8 matrix, matrix index
  const int r0 = lane >> 2, c2 = (lane & 3) * 2;

  auto load_q = [&](const uint8_t* qs) {
    if constexpr (!QF32) {
#pragma unroll
      for (int k2 = 0; k2 < C::KS; k2 += 2) {
        const int d0 = (k2 + (lm >> 1)) * 16 + ((lm & 1) << 3);
        ldsm_x4(smem_u32(qs + (lr * D + d0) * 2), qf[k2][0], qf[k2][1], qf[k2 + 1][0], qf[k2 + 1][1]);
      }
    } else {
      const float* qv = reinterpret_cast<const float*>(qs);
#pragma unroll
      for (int kk = 0; kk < C::KS; ++kk) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x = *reinterpret_cast<const float2*>(qv + r0 * D + kk * 16 + h * 8 + c2);
          const uint32_t hi = pack2<KT>(x.x, x.y);
          const float2 hf = unpack2<KT>(hi);
          qf[kk][h] = hi;
          ql[kk][h] = pack2<KT>(x.x - hf.x, x.y - hf.y);
        }
      }
    }
  };

  auto page_math = [&](const uint8_t* sb, int ntok) {
    const uint32_t kb = smem_u32(sb), vb = kb + C::PAGE_BYTES;
    float s[C::MT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
      s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < C::KS; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + swz<C::BOX_BYTES>(mt * 16 + lr + ((lm & 1) << 3), kk * 16 + ((lm >> 1) << 3)), a0, a1, a2, a3);
        Mma<KT>::run(s[mt], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
        if constexpr (QF32) Mma<KT>::run(s[mt], a0, a1, a2, a3, ql[kk][0], ql[kk][1]);
      }
    }
    // scores in log2 units; tokens past the end of the partition are -inf
    float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool ok = mt * 16 + r0 + 8 * h < ntok;
        s[mt][2 * h] = ok ? s[mt][2 * h] * p.scale_log2 : -CUDART_INF_F;
        s[mt][2 * h + 1] = ok ? s[mt][2 * h + 1] * p.scale_log2 : -CUDART_INF_F;
        mx0 = fmaxf(mx0, s[mt][2 * h]);
        mx1 = fmaxf(mx1, s[mt][2 * h + 1]);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, o));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float al0 = fast_exp2(m_run[0] - mn0), al1 = fast_exp2(m_run[1] - mn1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    l_run[0] *= al0;
    l_run[1] *= al1;
#pragma unroll
    for (int dt = 0; dt < C::KS; ++dt) {
      acc[dt][0] *= al0;
      acc[dt][1] *= al1;
      acc[dt][2] *= al0;
      acc[dt][3] *= al1;
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
      const uint32_t plo = pack2<KT>(fast_exp2(s[mt][0] - mn0), fast_exp2(s[mt][1] - mn1));
      const uint32_t phi = pack2<KT>(fast_exp2(s[mt][2] - mn0), fast_exp2(s[mt][3] - mn1));
      const float2 f0 = unpack2<KT>(plo), f1 = unpack2<KT>(phi);
      l_run[0] += f0.x + f1.x;  // the sum uses the rounded weights the MMA sees
      l_run[1] += f0.y + f1.y;
      const uint32_t b0 = movmatrix_t(plo), b1 = movmatrix_t(phi);
      // V rows past the end may hold anything (even NaN): zero them, 0 * NaN would poison
      const int tk = mt * 16 + c2;
      const uint32_t mlo = (tk < ntok ? 0x0000ffffu : 0u) | (tk + 1 < ntok ? 0xffff0000u : 0u);
      const uint32_t mhi = (tk + 8 < ntok ? 0x0000ffffu : 0u) | (tk + 9 < ntok ? 0xffff0000u : 0u);
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vb + swz<C::BOX_BYTES>(mt * 16 + lr + ((lm >> 1) << 3), dt * 16 + ((lm & 1) << 3)), a0, a1, a2, a3);
        if (ntok < BS) {
          a0 &= mlo;
          a1 &= mlo;
          a2 &= mhi;
          a3 &= mhi;
        }
        Mma<KT>::run(acc[dt], a0, a1, a2, a3, b0, b1);
      }
    }
  };

  auto finalize = [&](int seq, int part, int kvh, bool single) {
    float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(FULL, l0, o);
      l1 += __shfl_xor_sync(FULL, l1, o);
    }
    const int g0 = c2, g1 = c2 + 1;
    const int hq0 = kvh * G + g0, hq1 = hq0 + 1;
    const float nan = CUDART_NAN_F;
    if (single) {
      const float i0 = poisoned ? nan : 1.f / l0, i1 = poisoned ? nan : 1.f / l1;
      const int64_t o0 = (static_cast<int64_t>(seq) * Hq + hq0) * D, o1 = o0 + D;
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        const int d = dt * 16 + r0;
        if (g0 < G) {
          store_out(p.out, o0 + d, acc[dt][0] * i0, p.out_dtype);
          store_out(p.out, o0 + d + 8, acc[dt][2] * i0, p.out_dtype);
        }
        if (g1 < G) {
          store_out(p.out, o1 + d, acc[dt][1] * i1, p.out_dtype);
          store_out(p.out, o1 + d + 8, acc[dt][3] * i1, p.out_dtype);
        }
      }
    } else {
      const int64_t pidx = static_cast<int64_t>(seq) * p.max_parts + part;
      float* pa0 = p.part_acc + (pidx * Hq + hq0) * D;
      float* pa1 = pa0 + D;
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) {
        const int d = dt * 16 + r0;
        if (g0 < G) {
          pa0[d] = poisoned ? nan : acc[dt][0];
          pa0[d + 8] = poisoned ? nan : acc[dt][2];
        }
        if (g1 < G) {
          pa1[d] = poisoned ? nan : acc[dt][1];
          pa1[d + 8] = poisoned ? nan : acc[dt][3];
        }
      }
      if (lane < 4) {
        if (g0 < G) p.part_ml[pidx * Hq + hq0] = poisoned ? make_float2(0.f, nan) : make_float2(m_run[0], l0);
        if (g1 < G) p.part_ml[pidx * Hq + hq1] = poisoned ? make_float2(0.f, nan) : make_float2(m_run[1], l1);
      }
    }
  };

  auto consume = [&]() -> bool {
    const int slot = static_cast<int>(n_cons % C::NSLOT);
    // every lane waits (acquire); the vote keeps the warp together if a wait gives up
    const bool ready = mbar_wait_bounded(&bars[slot], (n_cons / C::NSLOT) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready)) return false;
    const int4 mt = meta[slot];
    const int ntok = mt.w >> 8, flags = mt.w & 0xff;
    const uint8_t* sb = ring + slot * C::SLOT_BYTES;
    if (flags & F_FIRST) {
      m_run[0] = m_run[1] = -CUDART_INF_F;
      l_run[0] = l_run[1] = 0.f;
#pragma unroll
      for (int dt = 0; dt < C::KS; ++dt) acc[dt][0] = acc[dt][1] = acc[dt][2] = acc[dt][3] = 0.f;
      poisoned = (flags & F_BAD) != 0;
      if (!poisoned) load_q(sb + 2 * C::PAGE_BYTES);
    }
    if (!poisoned) page_math(sb, ntok);
    if (flags & F_LAST) finalize(mt.x, mt.y, mt.z, (flags & F_SINGLE) != 0);
    ++n_cons;
    return true;
  };

  for (int s = 0; s < C::NSLOT; ++s)
    if (!fetch()) break;
  bool ok = true;
  while (n_cons < n_fetch) {
    if (!consume()) {
      ok = false;
      break;
    }
    __syncwarp();  // every lane is done reading the slot before lane 0 refills it
    fetch();
  }
  if (!ok) {
    if (lane == 0) record_error(DEV_TIMEOUT);
    // let the copies still in flight into this warp's slots land before the CTA exits
    for (uint32_t n = n_cons; n < n_fetch; ++n)
      mbar_wait_bounded(&bars[n % C::NSLOT], (n / C::NSLOT) & 1u, kWaitLimit);
  }
}

// ------------------------------------------------------------------------------ reduce
// One CTA per (sequence, KV head): merges the partitions of the G query heads.
__global__ void __launch_bounds__(128) pa_decode_reduce_kernel(const DecodeParams p) {
  const int seq = blockIdx.x, kvh = blockIdx.y;
  const int np = p.seq_nparts[seq];
  if (np == 1) return;  // written directly by the partition kernel
  const int G = p.group, D = p.head_dim, Hq = p.num_q_heads;
  const int64_t base = static_cast<int64_t>(seq) * p.max_parts;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, d = e - g * D, hq = kvh * G + g;
    float r;
    if (np == 0) {
      r = 0.f;
    } else if (np < 0) {
      r = CUDART_NAN_F;
    } else {
      float M = -CUDART_INF_F;
      for (int k = 0; k < np; ++k) M = fmaxf(M, p.part_ml[(base + k) * Hq + hq].x);
      float num = 0.f, den = 0.f;
      for (int k = 0; k < np; ++k) {
        const float2 ml = p.part_ml[(base + k) * Hq + hq];
        const float w = fast_exp2(ml.x - M);
        num += w * p.part_acc[((base + k) * Hq + hq) * D + d];
        den += w * ml.y;
      }
      r = num / den;
    }
    store_out(p.out, (static_cast<int64_t>(seq) * Hq + hq) * D + d, r, p.out_dtype);
  }
}

}  // namespace pa
