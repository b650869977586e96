// pa_decode_tc.cuh -- the partition kernel for wide work items on the 5th-generation tensor cores.
//
// Items with 9 to 32 query rows per KV head (several query tokens of a sequence, or the members of
// a shared prefix) carry 2-4x decode's math per K/V byte.  The kernel works on chunks of 8 pages
// (128 tokens) of one item, in the transposed form, so that both products have M = 128 with no
// padding and the softmax spreads over 128 threads:
//   S^T = K . Q^T     tcgen05.mma, M = 128 tokens, N = the item's query rows (16 or 32),
//                     K = head_dim; A = the chunk's K rows (TMA-staged, 128-byte swizzle),
//                     B = the query rows (written swizzled by the producer), D in tensor memory
//   softmax           thread t of the 128 consumer threads owns token t of the chunk (TMEM lane t)
//                     and holds, per query row, the running maximum and its own partial row sum;
//                     the maximum is raised (a CTA-wide vote) only when a score exceeds it by more
//                     than 2^8, and the O columns are then rescaled in tensor memory
//   O^T += V^T . P^T  tcgen05.mma per page, M = head_dim, N = query rows, K = 16 tokens;
//                     A = the staged V page read in place (MN-major), B = P^T in shared memory
// At the item's end the partial row sums are reduced across the 128 threads and thread d writes
// element d of every output row (coalesced).  The MMAs are issued by one thread and complete on
// mbarriers; the O product also releases the chunk's buffer to the producer.  The warp-MMA kernel
// of pa_decode.cuh is the default for these items (faster on B200); this one is chosen with
// pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_TCGEN05).
//
// CTA (one per SM): 3 chunk buffers of 64 KB; warps 0-3 run the softmax and the output (TMEM lane
// quarters 0-3), warp 4 produces (the work list, TMA for K/V, plain loads for the query rows),
// warp 5 issues every MMA.  Block size 16, head_dim 128, 16-bit cache and query.
#pragma once

#include "pa_decode.cuh"

namespace pa {

// ---------------------------------------------------------------- tcgen05 / tensor memory
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// generic-proxy writes to shared memory become visible to the tensor core's (async-proxy) reads
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] = A[smem] . B[smem] (+ D when accumulate)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// the mbarrier gets one arrival when every tcgen05 operation this thread issued before has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Shared-memory matrix descriptor (sm_100): start address, leading / stride byte offsets (all in
// 16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with fp32 accumulation: operand type (0 f16, 1 bf16),
// A / B major-ness (0 K-major, 1 MN-major), M and N.
__host__ __device__ constexpr uint32_t umma_idesc(uint32_t ab_type, uint32_t a_mn, uint32_t b_mn, uint32_t M,
                                                  uint32_t N) {
  return (1u << 4) | (ab_type << 7) | (ab_type << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// ---------------------------------------------------------------- helpers
// named barrier of the consumer warps, reducing a predicate (each warp reconverges first: the
// barrier instructions are warp-aligned)
__device__ __forceinline__ bool bar_and(bool v, int id, int nthreads) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool bar_or(bool v, int id, int nthreads) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync(int id, int nthreads) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
// N consecutive 32-bit TMEM columns of this thread's lane
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&v)[N]) {
  static_assert(N % 16 == 0, "columns");
#pragma unroll
  for (int i = 0; i < N / 16; ++i) tmem_ld16(taddr + 16 * i, *reinterpret_cast<uint32_t(*)[16]>(&v[16 * i]));
}
template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N / 16; ++i) tmem_st16(taddr + 16 * i, *reinterpret_cast<const uint32_t(*)[16]>(&v[16 * i]));
}

// ---------------------------------------------------------------- configuration
template <typename KT, int N>
struct TcCfg {
  static_assert(N == 16 || N == 32, "query rows per item");
  static constexpr int BS = 16, D = 128, QE = 2;
  static constexpr int CH = 8;                             // pages per chunk: 128 tokens
  static constexpr int NCH = 3;                            // chunk buffers
  static constexpr int BOX = BS * 128;                     // one TMA box: 16 rows x 128 bytes
  static constexpr int KH_BYTES = CH * BOX;                // one 64-element half of the chunk's K rows
  static constexpr int VPAGE = 2 * BOX;                    // a V page: two halves
  static constexpr int CHUNK_BYTES = 2 * KH_BYTES + CH * VPAGE;
  static constexpr int OPB = 2 * N * 128;                  // Q or P^T operand: 2 halves of N rows x 128 bytes
  static constexpr int QN = 2;                             // query buffers
  static constexpr int OFF_Q = NCH * CHUNK_BYTES;
  static constexpr int OFF_P = OFF_Q + QN * OPB;
  static constexpr int OFF_BAR = OFF_P + OPB;
  // mbarriers: chunk full / empty, query buffer free, S^T buffer full / free, P^T full, O product
  // done, final drain of the tensor pipe
  static constexpr int B_FULL = 0, B_EMPTY = NCH, B_QFREE = 2 * NCH, B_SFULL = B_QFREE + QN, B_SFREE = B_SFULL + 2,
                       B_PFULL = B_SFREE + 2, B_ODONE = B_PFULL + 1, B_FIN = B_ODONE + 1, NBAR = B_FIN + 1;
  static constexpr int OFF_META = OFF_BAR + ((NBAR * 8 + 15) & ~15);
  static constexpr int OFF_RED = OFF_META + NCH * 32;
  // reductions: per-warp partials [4][N], row maxima [N], rescale factors [N], output scales [N],
  // output offsets [N] (int64)
  static constexpr int OFF_MISC = OFF_RED + 7 * N * 4 + N * 8;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
  // warps 0-3 consume (softmax, output), warp 4 loads, warp 5 issues the MMAs
  static constexpr int NCONS = 128, NTHREADS = NCONS + 64;
  // TMEM columns: O^T, then two S^T buffers
  static constexpr uint32_t TM_COLS = 3 * N <= 64 ? 64 : 128, TM_O = 0, TM_S = N;
  static constexpr uint32_t AB = std::is_same<KT, __nv_bfloat16>::value ? 1u : 0u;
  static constexpr uint32_t IDESC_S = umma_idesc(AB, 0, 0, 128, N);  // K (K-major) . Q^T (K-major)
  static constexpr uint32_t IDESC_O = umma_idesc(AB, 1, 0, 128, N);  // V^T (MN-major) . P^T (K-major)
  static_assert(CHUNK_BYTES % 1024 == 0 && OFF_Q % 1024 == 0 && OPB % 1024 == 0 && (N * 128) % 1024 == 0,
                "128-byte swizzle atoms");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// ---------------------------------------------------------------- producer (warp 4)
// The loads that place an item (its work-list entry, block-table row, sequence length and query
// rows) form a chain of dependent global reads.  The producer runs it ahead of the ring: while the
// chunks of item k are issued, the entry of item k + 2 and the rest of item k + 1 are in flight.
template <int QPL>
struct TcItemLoads {
  bool valid;
  WorkItem it;
  int kvh, bt, rel0;
  bool mismatch;
  uint4 qv[QPL];
};

template <typename C, int N>
__device__ __forceinline__ void tc_produce(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                           uint8_t* smem, uint64_t* bars, int4* meta, volatile int* abort_flag,
                                           int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int BS = C::BS, D = C::D, QPL = N / 2;  // query chunks (16 bytes) per lane
  uint64_t* full = bars + C::B_FULL;
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* qfree = bars + C::B_QFREE;
  const int G = p.group, Hkv = p.num_kv_heads, Hq = p.num_q_heads, T = p.qtok;
  const unsigned total = p.counters[1] * static_cast<unsigned>(Hkv);
  const uint64_t pol = policy_evict_first();
  const uint8_t* qsrc = static_cast<const uint8_t*>(p.q);
  uint32_t nchunks = 0, items = 0;
  bool stop = false;
  auto acquire = [&](int c) -> bool {  // wait until the chunk buffer c was released
    if (nchunks < C::NCH) return true;
    const bool ok = mbar_wait_bounded(&empty[c], ((nchunks / C::NCH) - 1) & 1u, kWaitLimit);
    return __all_sync(FULL, ok && !*abort_flag);
  };
  auto claim = [&]() -> unsigned {  // lane 0's claim; read (broadcast) one item later
    unsigned w = 0;
    if (lane == 0) w = atomicAdd(&p.counters[0], 1u);
    return w;
  };
  // q / d for 0 <= q < 1024 and 1 <= d <= 64: (q * ceil(2^16 / d)) >> 16 is exact there
  const uint32_t inv_g = (65536u + G - 1) / G;
  auto entry = [&](unsigned w) -> WorkItem {
    return w < total ? p.items[w / Hkv] : WorkItem{0, 0, 0, 0, 0, 1, 0, 0};
  };
  // issue every load of item w (entry `it`); nothing here waits for them
  auto issue_loads = [&](unsigned w, const WorkItem& it, TcItemLoads<QPL>& L) {
    L.valid = w < total;
    L.it = it;
    L.kvh = static_cast<int>(w % Hkv);
    L.bt = 0;
    L.mismatch = false;
    L.rel0 = 0;
    if (!L.valid) return;
    const int members = (it.pm >> 16) & 0xff;
    const int npages = (it.tok1 - it.tok0 + BS - 1) / BS;
    if (lane < npages) {
      const int64_t col = it.tok0 / BS + lane;
      L.bt = p.block_tables[static_cast<int64_t>(it.seq) * p.max_blocks_per_seq + col];
      for (int m = 1; m < members; ++m)  // the members of a shared item must hold the same blocks
        L.mismatch |= p.block_tables[static_cast<int64_t>(it.seq + m) * p.max_blocks_per_seq + col] != L.bt;
    }
    // key positions relative to the item's first query token, at position len - T + t0
    if (T > 1) L.rel0 = it.tok0 - (p.seq_lens[it.seq] - T + it.t0);
    const int ncol = members * it.tq * G;
    const uint32_t inv_tq = (65536u + it.tq - 1) / it.tq;
#pragma unroll
    for (int k = 0; k < QPL; ++k) {
      const int idx = lane + 32 * k;  // row idx / 16, 16-byte chunk idx % 16
      if (idx < ncol * 16) {
        const int r = idx >> 4, mt = static_cast<int>((r * inv_g) >> 16), g = r - mt * G;
        const int m = static_cast<int>((mt * inv_tq) >> 16), t = it.t0 + mt - m * it.tq;
        const int64_t qrow = (static_cast<int64_t>(it.seq + m) * T + t) * Hq + L.kvh * G + g;
        L.qv[k] = __ldg(reinterpret_cast<const uint4*>(qsrc + (qrow * D + (idx & 15) * 8) * C::QE));
      }
    }
  };

  TcItemLoads<QPL> cur, nxt;
  const unsigned c0 = claim();
  const unsigned c1 = claim();
  const unsigned w0 = __shfl_sync(FULL, c0, 0);
  issue_loads(w0, entry(w0), cur);
  unsigned w1 = __shfl_sync(FULL, c1, 0);
  WorkItem it1 = entry(w1);
  unsigned c2 = claim();
  while (cur.valid) {
    issue_loads(w1, it1, nxt);  // item k + 1
    w1 = __shfl_sync(FULL, c2, 0);
    it1 = entry(w1);  // item k + 2
    c2 = claim();     // item k + 3

    // ---- item k
    const WorkItem& it = cur.it;
    const int kvh = cur.kvh;
    const int part = it.pm & 0xffff, members = (it.pm >> 16) & 0xff;
    const int tok0 = it.tok0, tok1 = it.tok1;
    const int npages = (tok1 - tok0 + BS - 1) / BS;
    const int rows = members * it.tq, ncol = rows * G;
    bool bad = lane < npages && (cur.bt < 0 || cur.bt >= p.num_blocks);
    bad = __any_sync(FULL, bad);
    const bool mismatch = __any_sync(FULL, cur.mismatch);
    if (lane == 0) {
      if (bad) record_error(DEV_BAD_BLOCK_ID);
      if (mismatch) record_error(DEV_BAD_PREFIX);
    }
    bad |= mismatch;
    const uint32_t qb = items % C::QN;
    if (items >= C::QN) {  // the tensor core is done with the query rows of item `items - QN`
      const bool ok = mbar_wait_bounded(&qfree[qb], ((items / C::QN) - 1) & 1u, kWaitLimit);
      if (!__all_sync(FULL, ok && !*abort_flag)) {
        stop = true;
        break;
      }
    }
    if (!bad) {
      // query row r -> half h, row r, 16-byte chunk ch at h * N * 128 + r * 128 + ((ch ^ (r & 7)) << 4):
      // the 128-byte-swizzled K-major B operand
      uint8_t* qdst = smem + C::OFF_Q + qb * C::OPB;
#pragma unroll
      for (int k = 0; k < QPL; ++k) {
        const int idx = lane + 32 * k, r = idx >> 4, c16 = idx & 15;
        if (idx < ncol * 16)
          *reinterpret_cast<uint4*>(qdst + (c16 >> 3) * (N * 128) + r * 128 + (((c16 & 7) ^ (r & 7)) << 4)) = cur.qv[k];
      }
      fence_proxy_async_smem();
    }
    __syncwarp();
    const int nch = (npages + C::CH - 1) / C::CH;
    for (int cc = 0; cc < nch; ++cc) {
      const int c = static_cast<int>(nchunks % C::NCH);
      if (!acquire(c)) {
        stop = true;
        break;
      }
      const int pg0 = cc * C::CH, npg = min(C::CH, npages - pg0);
      const int phys = __shfl_sync(FULL, cur.bt, (pg0 + lane) & 31);
      if (lane == 0) {
        const int ntok_last = min(BS, tok1 - (tok0 + (pg0 + npg - 1) * BS));
        const int flags = (cc == 0 ? F_FIRST : 0) | (cc == nch - 1 ? F_LAST : 0) | (bad ? F_BAD : 0) |
                          ((it.pm & WI_DIRECT) ? F_DIRECT : 0);
        meta[2 * c] = make_int4(it.seq, part, kvh | (npg << 8) | (rows << 16) | (flags << 24), cur.rel0 + pg0 * BS);
        meta[2 * c + 1] = make_int4(it.t0, ntok_last, static_cast<int>(qb), 0);
        if (bad)
          mbar_arrive(&full[c]);
        else
          mbar_arrive_expect_tx(&full[c], static_cast<uint32_t>(npg * 2 * C::VPAGE));
      }
      __syncwarp();  // the expected byte count is set before any copy can complete
      // one box per lane: page lane / 4, K half 0 / K half 1 / V half 0 / V half 1
      const int lp = lane >> 2, lh = lane & 1;
      const bool lv = (lane & 2) != 0;
      const int lphys = __shfl_sync(FULL, phys, lp);
      if (!bad && lp < npg) {
        uint8_t* cb = smem + c * C::CHUNK_BYTES;
        uint8_t* dst = lv ? cb + 2 * C::KH_BYTES + lp * C::VPAGE + lh * C::BOX : cb + lh * C::KH_BYTES + lp * C::BOX;
        tma_load_3d(dst, lv ? &tmv : &tmk, 0, kvh * 2 + lh, lphys * BS, &full[c], pol);
      }
      ++nchunks;
    }
    if (stop) break;
    ++items;
    cur = nxt;
  }
  if (!stop) {  // tell the other roles there is no more work
    const int c = static_cast<int>(nchunks % C::NCH);
    if (acquire(c)) {
      if (lane == 0) {
        meta[2 * c] = make_int4(0, 0, F_END << 24, 0);
        mbar_arrive(&full[c]);
      }
    } else {
      stop = true;
    }
  }
  if (stop) {
    if (lane == 0) {
      record_error(DEV_TIMEOUT);
      *abort_flag = 1;
    }
    // copies this warp issued may still be landing: wait for them before the CTA exits
    for (uint32_t k = nchunks > C::NCH ? nchunks - C::NCH : 0; k < nchunks; ++k)
      mbar_wait_bounded(&full[k % C::NCH], (k / C::NCH) & 1u, kWaitLimit);
  }
}

// ---------------------------------------------------------------- MMA issue (warp 5)
// For chunk n: S^T(n) as soon as the chunk is in and its S^T buffer is free; O^T += V^T . P^T(n)
// once the consumers have written P^T(n).  S^T(n + 1) is issued before O(n), so that it runs
// during chunk n's softmax.
template <typename C, int N>
__device__ __forceinline__ void tc_mma(uint8_t* smem, uint64_t* bars, const int4* meta, volatile int* abort_flag,
                                       uint32_t tm, int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int D = C::D;
  uint64_t* full = bars + C::B_FULL;
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* qfree = bars + C::B_QFREE;
  uint64_t* s_full = bars + C::B_SFULL;
  uint64_t* s_free = bars + C::B_SFREE;
  uint64_t* p_full = bars + C::B_PFULL;
  uint64_t* o_done = bars + C::B_ODONE;
  struct Chunk {
    int c, npg, qb;
    bool end, poisoned, first, last;
  };
  uint32_t ns = 0, np = 0;  // S^T and O products issued
  bool item_bad = false;
  int item_qb = 0;
  bool ok = true;
  auto prepare = [&](uint32_t k) -> Chunk {
    Chunk ch{static_cast<int>(k % C::NCH), 0, 0, true, false, false, false};
    const bool ready = mbar_wait_bounded(&full[ch.c], (k / C::NCH) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready && !*abort_flag)) {
      ok = false;
      return ch;
    }
    const int4 m0 = meta[2 * ch.c], m1 = meta[2 * ch.c + 1];
    const int flags = (m0.z >> 24) & 0xff;
    if (flags & F_END) return ch;
    ch.end = false;
    ch.first = (flags & F_FIRST) != 0;
    ch.last = (flags & F_LAST) != 0;
    if (ch.first) {
      item_bad = (flags & F_BAD) != 0;
      item_qb = m1.z;
    }
    ch.poisoned = item_bad;
    ch.qb = item_qb;
    ch.npg = (m0.z >> 8) & 0xff;
    if (!ch.poisoned) {
      const uint32_t b = ns & 1u;
      if (ns >= 2) {  // the consumers have read S^T(ns - 2) out of this buffer
        const bool fr = mbar_wait_bounded(&s_free[b], ((ns >> 1) - 1) & 1u, kWaitLimit);
        if (!__all_sync(FULL, fr)) {
          ok = false;
          ch.end = true;
          return ch;
        }
      }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + ch.c * C::CHUNK_BYTES);
        const uint32_t qa = smem_u32(smem + C::OFF_Q + ch.qb * C::OPB);
#pragma unroll
        for (int k2 = 0; k2 < D / 16; ++k2) {
          const uint32_t a = kb + (k2 >> 2) * C::KH_BYTES + (k2 & 3) * 32;
          const uint32_t bq = qa + (k2 >> 2) * (N * 128) + (k2 & 3) * 32;
          umma_ss(tm + C::TM_S + b * N, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(bq, 16, 1024), C::IDESC_S,
                  k2 > 0);
        }
        umma_commit(&s_full[b]);
        if (ch.last) umma_commit(&qfree[ch.qb]);  // the query rows are read once the item's last S^T is done
      }
      __syncwarp();
      ++ns;
    }
    return ch;
  };

  // chunk k is in (no waiting)
  auto arrived = [&](uint32_t k) -> bool {
    uint32_t done = 0;
    if (lane == 0) done = mbar_test(&full[k % C::NCH], (k / C::NCH) & 1u) ? 1u : 0u;
    return __shfl_sync(FULL, done, 0) != 0;
  };

  uint32_t n = 0;
  Chunk cur = prepare(0);
  while (ok && !cur.end) {
    // S^T(n + 1) goes first when its chunk is already in; O(n) never waits for the next chunk
    bool have_next = false;
    Chunk nxt;
    if (arrived(n + 1)) {
      nxt = prepare(n + 1);
      have_next = true;
      if (!ok) break;
    }
    if (!cur.poisoned) {
      const bool pf = mbar_wait_bounded(p_full, np & 1u, kWaitLimit);
      if (!__all_sync(FULL, pf)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t vb = smem_u32(smem + cur.c * C::CHUNK_BYTES + 2 * C::KH_BYTES);
        const uint32_t pb = smem_u32(smem + C::OFF_P);
        for (int j = 0; j < cur.npg; ++j) {
          const uint64_t a = smem_desc_sw128(vb + j * C::VPAGE, C::BOX, 1024);
          const uint64_t b = smem_desc_sw128(pb + (j >> 2) * (N * 128) + (j & 3) * 32, 16, 1024);
          umma_ss(tm + C::TM_O, a, b, C::IDESC_O, (cur.first && j == 0) ? 0u : 1u);
        }
        umma_commit(o_done);
        umma_commit(&empty[cur.c]);  // the chunk buffer is free once these products are done
      }
      __syncwarp();
      ++np;
    } else if (lane == 0) {
      mbar_arrive(&empty[cur.c]);
      if (cur.last) mbar_arrive(&qfree[cur.qb]);
    }
    if (!have_next) {
      nxt = prepare(n + 1);
      if (!ok) break;
    }
    cur = nxt;
    ++n;
  }
  if (!ok && lane == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
  // every product issued here completes before the tensor memory is released
  if (lane == 0) {
    umma_commit(bars + C::B_FIN);
  }
  __syncwarp();
  mbar_wait_bounded(bars + C::B_FIN, 0u, kWaitLimit);
}

// ---------------------------------------------------------------- kernel
template <typename KT, int N, bool CAUSAL>
__global__ void __launch_bounds__(TcCfg<KT, N>::NTHREADS, 1)
    pa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const DecodeParams p) {
  using C = TcCfg<KT, N>;
  constexpr int D = C::D, NC = C::NCONS;
  constexpr int BAR_C = 1;     // named barrier of the consumer warps
  constexpr int BAR_EXIT = 2;  // consumers and the MMA warp, before the tensor memory is released

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [4][N] per-warp partials
  float* msm = red + 4 * N;                                  // [N] running row maxima
  float* asm_ = msm + N;                                     // [N] rescale factors
  float* fscale = asm_ + N;                                  // [N] output scale of each row
  int64_t* fofs = reinterpret_cast<int64_t*>(fscale + N);    // [N] output offset of each row
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NBAR; ++s) {
      // S^T free and P^T full: one arrival per consumer warp; a chunk buffer is free once the
      // consumer warps have read its meta and the MMA warp has finished with it (or skipped it)
      const bool four = s == C::B_SFREE || s == C::B_SFREE + 1 || s == C::B_PFULL;
      const bool empty = s >= C::B_EMPTY && s < C::B_EMPTY + C::NCH;
      mbar_init(&bars[s], four ? 4 : empty ? 5 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();  // the plan kernel's work list and counters are visible from here on

  if (warp == 4) {
    tc_produce<C, N>(p, tmk, tmv, smem, bars, meta, abort_flag, lane);
    return;
  }
  if (warp == 5) {
    tc_mma<C, N>(smem, bars, meta, abort_flag, tm, lane);
    tc_fence_before();
    bar_sync(BAR_EXIT, NC + 32);
    return;
  }

  // ============================== consumers (warps 0-3) ==============================
  constexpr unsigned FULL = 0xffffffffu;
  constexpr float kNone = -1e30f;  // running maximum of a row with no score yet (finite: no NaN from -inf - -inf)
  uint64_t* full = bars + C::B_FULL;
  uint64_t* s_full = bars + C::B_SFULL;
  uint64_t* s_free = bars + C::B_SFREE;
  uint64_t* p_full = bars + C::B_PFULL;
  uint64_t* o_done = bars + C::B_ODONE;
  const int ct = threadIdx.x;  // token of the chunk (S^T lane), element of head_dim (O^T lane)
  const uint32_t tl = tm + (static_cast<uint32_t>(warp * 32) << 16);  // this warp's lane quarter
  uint8_t* pbuf = smem + C::OFF_P;

  const int G = p.group, Hq = p.num_q_heads, T = p.qtok, HV = T * Hq;
  const float sl = p.scale_log2;
  uint32_t n = 0, ns = 0, o_phase = 0;
  bool o_pending = false, ok = true;
  float m[N], lp[N];
  int ncol = 0, item_t0 = 0;
  bool poisoned = false, o_fresh = true;

  // completion of the last O product
  auto wait_o = [&]() -> bool {
    bool fin = true;
    if (o_pending) {
      fin = mbar_wait_bounded(o_done, o_phase, kWaitLimit);
      o_phase ^= 1u;
      o_pending = false;
      tc_fence_after();
    }
    return fin;
  };

  while (true) {
    const int c = static_cast<int>(n % C::NCH);
    const bool ready = mbar_wait_bounded(&full[c], (n / C::NCH) & 1u, kWaitLimit);
    if (!bar_and(ready && !*abort_flag, BAR_C, NC)) {
      ok = false;
      break;
    }
    const int4 m0 = meta[2 * c], m1 = meta[2 * c + 1];
    const int flags = (m0.z >> 24) & 0xff;
    if (flags & F_END) break;
    if (flags & F_FIRST) {
      poisoned = (flags & F_BAD) != 0;
      ncol = ((m0.z >> 16) & 0xff) * G;
      item_t0 = m1.x;
      o_fresh = true;
#pragma unroll
      for (int r = 0; r < N; ++r) {
        m[r] = kNone;
        lp[r] = 0.f;
      }
      if (ct < N) msm[ct] = kNone;  // read only after the next barrier
    }
    const int npg = (m0.z >> 8) & 0xff, ntok_last = m1.y;
    const bool last = (flags & F_LAST) != 0;
    uint8_t* cb = smem + c * C::CHUNK_BYTES;

    if (!poisoned) {
      const int pg = ct >> 4, ti = ct & 15;
      const bool valid = pg < npg && (pg < npg - 1 || ti < ntok_last);
      if (pg == npg - 1 && ti >= ntok_last) {
        // V rows past the end of the item may hold anything (even NaN) and would meet zero
        // weights in the MMA: zero this token's row
        uint8_t* vrow = cb + 2 * C::KH_BYTES + pg * C::VPAGE + ti * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int q = 0; q < 8; ++q) *reinterpret_cast<uint4*>(vrow + h * C::BOX + q * 16) = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
      }
      const uint32_t b = ns & 1u;
      bool good = mbar_wait_bounded(&s_full[b], (ns >> 1) & 1u, kWaitLimit);
      tc_fence_after();
      uint32_t sr[N];
      tmem_ldn<N>(tl + C::TM_S + b * N, sr);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      ++ns;

      // scores in log2 units, -inf where masked: rows r < ncol; with several query tokens, row r
      // (query token r / G) sees keys at relative positions <= r / G, i.e. r >= rel * G
      const int lo = CAUSAL && T > 1 ? (m0.w + ct) * G : 0;
      float x[N];
      bool big = false;
#pragma unroll
      for (int r = 0; r < N; ++r) {
        const bool keep = valid && r < ncol && r >= lo;
        x[r] = keep ? __uint_as_float(sr[r]) * sl : -CUDART_INF_F;
        big |= x[r] > m[r] + kRescaleThreshold;
      }
      // the previous O product is done: O may be rescaled and P^T overwritten
      good = wait_o() && good;
      if (bar_or(big || !good, BAR_C, NC)) {
        if (!bar_and(good, BAR_C, NC)) {
          ok = false;
          break;
        }
        big = bar_or(big, BAR_C, NC);
      }
      if (big) {  // uniform here
        // raise the maximum of every row whose chunk maximum exceeds it by more than the
        // threshold: a butterfly leaves row lane % N's warp maximum in each lane, thread r < N
        // decides row r
        float v[N];
#pragma unroll
        for (int r = 0; r < N; ++r) v[r] = x[r];
        if (N == 16) {
#pragma unroll
          for (int r = 0; r < N; ++r) v[r] = fmaxf(v[r], __shfl_xor_sync(FULL, v[r], 16));
        }
#pragma unroll
        for (int s2 = N / 2; s2 >= 1; s2 >>= 1) {
          const bool upper = (lane & s2) != 0;
#pragma unroll
          for (int i = 0; i < s2; ++i) {
            const float send = upper ? v[i] : v[i + s2];
            const float keep = upper ? v[i + s2] : v[i];
            v[i] = fmaxf(keep, __shfl_xor_sync(FULL, send, s2));
          }
        }
        if (lane < N) red[warp * N + lane] = v[0];
        bar_sync(BAR_C, NC);
        if (ct < N) {
          const float mo = msm[ct];
          const float cm = fmaxf(fmaxf(red[ct], red[N + ct]), fmaxf(red[2 * N + ct], red[3 * N + ct]));
          float a = 1.f;
          if (cm > mo + kRescaleThreshold) {
            a = fast_exp2(mo - cm);  // 0 for a row without scores so far
            msm[ct] = cm;
          }
          asm_[ct] = a;
        }
        bar_sync(BAR_C, NC);
        bool rescale = false;
        float alpha[N];
#pragma unroll
        for (int r = 0; r < N; ++r) {
          alpha[r] = asm_[r];
          m[r] = msm[r];
          lp[r] *= alpha[r];
          rescale |= alpha[r] != 1.f;
        }
        // (rescale is the same in every thread; O is idle: the previous product is done and this
        // chunk's is not issued before the consumers signal P^T)
        if (rescale && !o_fresh) {
          uint32_t ov[N];
          tmem_ldn<N>(tl + C::TM_O, ov);
          tc_wait_ld();
#pragma unroll
          for (int r = 0; r < N; ++r) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha[r]);
          tmem_stn<N>(tl + C::TM_O, ov);
          tc_wait_st();
        }
      }
      // P^T (K-major: row r = query row, 128 tokens in two 64-token halves, 128-byte swizzle)
      const uint32_t prow = smem_u32(pbuf) + (ct >> 6) * (N * 128) + (ct & 7) * 2;
      const int pch = (ct & 63) >> 3;
#pragma unroll
      for (int r = 0; r < N; r += 2) {
        const uint32_t pk = pack2<KT>(fast_exp2(x[r] - m[r]), fast_exp2(x[r + 1] - m[r + 1]));
        const float2 w2 = unpack2<KT>(pk);  // the weights the MMA sees
        lp[r] += w2.x;
        lp[r + 1] += w2.y;
        sts_u16(prow + r * 128 + ((pch ^ (r & 7)) << 4), static_cast<uint16_t>(pk & 0xffffu));
        sts_u16(prow + (r + 1) * 128 + ((pch ^ ((r + 1) & 7)) << 4), static_cast<uint16_t>(pk >> 16));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(p_full);
        mbar_arrive(&bars[C::B_EMPTY + c]);
      }
      o_pending = true;
      o_fresh = false;
    } else {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[C::B_EMPTY + c]);
    }

    if (last) {
      // output of the item: reduce the row sums over the 128 threads
      const bool good = wait_o();
      if (!bar_and(good, BAR_C, NC)) {
        ok = false;
        break;
      }
      const bool bad = poisoned || o_fresh;  // uniform
      float v[N];
#pragma unroll
      for (int r = 0; r < N; ++r) v[r] = lp[r];
      if (N == 16) {
#pragma unroll
        for (int r = 0; r < N; ++r) v[r] += __shfl_xor_sync(FULL, v[r], 16);
      }
#pragma unroll
      for (int s2 = N / 2; s2 >= 1; s2 >>= 1) {
        const bool upper = (lane & s2) != 0;
#pragma unroll
        for (int i = 0; i < s2; ++i) {
          const float send = upper ? v[i] : v[i + s2];
          const float keep = upper ? v[i + s2] : v[i];
          v[i] = keep + __shfl_xor_sync(FULL, send, s2);
        }
      }
      if (lane < N) red[warp * N + lane] = v[0];
      bar_sync(BAR_C, NC);
      const int seq = m0.x, part = m0.y & 0xffff, kvh = m0.z & 0xff;
      const bool direct = (flags & F_DIRECT) != 0;
      if (ct < ncol) {  // row ct: where it goes and how it is scaled
        const float l = red[ct] + red[N + ct] + red[2 * N + ct] + red[3 * N + ct];
        const int g = ct % G, mq = ct / G;
        const int mb = T > 1 ? 0 : mq, t = T > 1 ? item_t0 + mq : 0;
        const int vh = t * Hq + kvh * G + g;
        if (direct) {
          fofs[ct] = (static_cast<int64_t>(seq + mb) * HV + vh) * D;
          fscale[ct] = bad ? CUDART_NAN_F : p.v_scale / l;
        } else {
          const int64_t pidx = static_cast<int64_t>(seq + mb) * p.max_parts + part;
          fofs[ct] = (pidx * HV + vh) * D;
          fscale[ct] = bad ? CUDART_NAN_F : p.v_scale;
          __stcg(&p.part_ml[pidx * HV + vh], bad ? make_float2(0.f, CUDART_NAN_F) : make_float2(msm[ct], l));
        }
      }
      bar_sync(BAR_C, NC);
      uint32_t ov[N];
      if (!bad) {
        tmem_ldn<N>(tl + C::TM_O, ov);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int r = 0; r < N; ++r) ov[r] = 0u;
      }
      auto emit = [&](auto store) {
#pragma unroll
        for (int r = 0; r < N; ++r)
          if (r < ncol) store(fofs[r] + ct, __uint_as_float(ov[r]) * fscale[r]);
      };
      if (!direct)
        emit([&](int64_t i, float val) { __stcg(p.part_acc + i, val); });
      else if (p.out_dtype == DT_BF16)
        emit([&](int64_t i, float val) { static_cast<__nv_bfloat16*>(p.out)[i] = __float2bfloat16_rn(val); });
      else if (p.out_dtype == DT_F16)
        emit([&](int64_t i, float val) { static_cast<__half*>(p.out)[i] = __float2half_rn(val); });
      else
        emit([&](int64_t i, float val) { static_cast<float*>(p.out)[i] = val; });
      tc_fence_before();
      bar_sync(BAR_C, NC);  // red[], fofs[] and the O columns are reused by the next item
    }
    ++n;
  }
  if (!ok && ct == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
  tc_fence_before();
  bar_sync(BAR_EXIT, NC + 32);  // the MMA warp has drained the tensor pipe
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, C::TM_COLS);
  }
}

}  // namespace pa
