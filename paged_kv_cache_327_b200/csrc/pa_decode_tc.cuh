// pa_decode_tc.cuh -- the partition kernel for wide work items on the 5th-generation tensor cores.
//
// Items with several query rows per KV head (the query tokens of a sequence, or the members of a
// shared prefix: up to 64 rows) carry up to 8x decode's math per K/V byte.  The query rows sit on
// the M dimension of the products, so that every softmax reduction stays on the row's lane:
//   S = Q . K^T      tcgen05.mma, M = 64 query rows, N = 64 tokens (a chunk of 4 pages), K =
//                    head_dim; A = the item's query rows (TMA-staged once per item), B = the
//                    chunk's K rows (TMA-staged, 128-byte swizzle), D in tensor memory
//   softmax          an M = 64 product keeps 16 rows in each TMEM lane quarter; a warp reads all
//                    64 columns of its quarter's rows in the 16x256b shape, so every lane holds
//                    scores of two rows (a quad of lanes shares a row) and the rows' chunk maxima
//                    are agreed by shuffles in the quad; the maximum is raised (and the O rows
//                    rescaled in tensor memory) only when a score exceeds it by more than 2^8, and
//                    the weights P, rounded to the operand type, go to shared memory
//   O += P . V       tcgen05.mma per page, M = 64, N = head_dim, K = 16 tokens; A = P, B = the
//                    staged V page read in place (MN-major)
// Two groups of four softmax warps take the chunks (S products) in turn, so that two chunks are
// in the softmax at once.  Each group keeps its own online softmax over its chunks of an item --
// running maxima, row sums, and an O accumulator in tensor memory -- so neither waits for the
// other's maxima; the two states meet at the item's end, where the two warps of a lane quarter
// exchange (maximum, sum) per row and each writes half of the head_dim outputs of the quarter's 16
// rows.  S and O products are issued by two warps of their own, so that neither waits for the
// other's issue, and complete on mbarriers.  Buffers keep every stage busy: three S buffers, a P
// buffer per group, two query buffers and five chunk buffers of 32 KB in flight per SM.
//
// CTA (one per SM): warps 0-7 run the softmax and the output (warp w on TMEM lane quarter w % 4,
// the chunks whose S product index has the parity of w / 4; a quarter without the item's rows
// skips the arithmetic), warp 8 produces (the work list, TMA for the K/V pages and the query
// rows), warp 9 issues the S products, warp 10 the O products.
// Block size 16, head_dim 128, 16-bit cache and query.
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

// 16 TMEM lanes x 256 bits per repetition (8 columns of 32 bits): in each 8-column block j, thread t
// holds (lane t / 4, columns 8 j + 2 (t % 4), + 1) in registers 4 j, 4 j + 1 and (lane t / 4 + 8,
// the same columns) in 4 j + 2, 4 j + 3 -- the lanes counted from the address's lane field.
__device__ __forceinline__ void tmem_ld16x256_x4(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16x256_x4(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// N / 4 repetitions of the x4 form: N registers, columns 0 .. 2 N - 1 from the address
template <int N>
__device__ __forceinline__ void tmem_ld16x256(uint32_t taddr, uint32_t (&v)[N]) {
  static_assert(N % 16 == 0, "registers");
#pragma unroll
  for (int i = 0; i < N / 16; ++i)
    tmem_ld16x256_x4(taddr + 32 * i, *reinterpret_cast<uint32_t(*)[16]>(&v[16 * i]));
}
template <int N>
__device__ __forceinline__ void tmem_st16x256(uint32_t taddr, const uint32_t (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N / 16; ++i)
    tmem_st16x256_x4(taddr + 32 * i, *reinterpret_cast<const uint32_t(*)[16]>(&v[16 * i]));
}

// ---------------------------------------------------------------- helpers
// four 8x8 matrices of 16-bit elements to shared memory: register i of thread t holds row t / 4,
// columns 2 (t % 4) and + 1 of matrix i; threads 8 i .. 8 i + 7 give the addresses of its 8 rows
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}
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
template <typename KT>
struct TcCfg {
  static constexpr int BS = 16, D = 128;
  static constexpr int M = 64;                              // MMA rows: the item's query rows
  static constexpr int CH = 4;                              // pages per chunk
  static constexpr int CT = CH * BS;                        // tokens per chunk: N of S
  static constexpr int NCH = 5;                             // chunk buffers
  static constexpr int BOX = BS * 128;                      // one TMA box: 16 rows x 128 bytes
  static constexpr int KPAGE = 2 * BOX;                     // a K page: [row half][column block][8 rows][128 B]
  static constexpr int VPAGE = 2 * BOX;                     // a V page: [column block][16 rows][128 B]
  static constexpr int KC_BYTES = CH * KPAGE;               // the chunk's K rows
  static constexpr int CHUNK_BYTES = KC_BYTES + CH * VPAGE;
  static constexpr int QHALF = M * 128;                     // one 64-element half of the query rows
  static constexpr int QBUF = 2 * QHALF;
  static constexpr int QN = 2;                              // query buffers
  static constexpr int PBUF = M * 128;                      // P: M rows x 64 tokens (one swizzle atom wide)
  static constexpr int OFF_Q = NCH * CHUNK_BYTES;
  static constexpr int OFF_P = OFF_Q + QN * QBUF;
  static constexpr int OFF_BAR = OFF_P + 2 * PBUF;
  // mbarriers: chunk full / empty, query buffer free, S full / free, P full / free (the O product
  // that read it is done), O accumulators free (the item's output has been read), final drain,
  // the two softmax groups' item states [quarter][item parity]; and chunk meta written (before
  // its copies land)
  static constexpr int NSB = 3;  // S buffers: S products run up to NSB - 1 chunks ahead of the softmax
  static constexpr int B_FULL = 0, B_EMPTY = NCH, B_QFREE = 2 * NCH, B_SFULL = B_QFREE + QN, B_SFREE = B_SFULL + NSB,
                       B_PFULL = B_SFREE + NSB, B_PFREE = B_PFULL + 2, B_OFREE = B_PFREE + 2, B_FIN = B_OFREE + 1,
                       B_SUM = B_FIN + 1, B_META = B_SUM + 8, NBAR = B_META + NCH;
  static constexpr int OFF_META = OFF_BAR + ((NBAR * 8 + 15) & ~15);
  // exchange between the two softmax warps of a lane quarter: each group's (running maximum,
  // sum) of a row at the item's end, [item parity][group][M]
  static constexpr int OFF_XCH = OFF_META + NCH * 32;
  static constexpr int OFF_MISC = OFF_XCH + 2 * 2 * M * 8;
  static constexpr int SMEM_BYTES = 1024 + OFF_MISC + 16;
  // warps 0-7: softmax and output, warp 8 loads, warp 9 issues the S products, warp 10 the O products
  static constexpr int NSM = 256, W_LOAD = 8, W_S = 9, W_O = 10, NTHREADS = NSM + 96;
  static constexpr int HC = CT;  // chunk columns per softmax warp: all of them (groups alternate chunks)
  // TMEM columns: the two softmax groups' O accumulators (head_dim columns each), then NSB S
  // buffers (one chunk each)
  static constexpr uint32_t TM_COLS = 512, TM_O = 0, TM_S = 2 * D;
  static constexpr uint32_t AB = std::is_same<KT, __nv_bfloat16>::value ? 1u : 0u;
  static constexpr uint32_t IDESC_S = umma_idesc(AB, 0, 0, M, CT);  // Q (K-major) . K^T (K-major)
  static constexpr uint32_t IDESC_O = umma_idesc(AB, 0, 1, M, D);   // P (K-major) . V (MN-major)
  static_assert(32 % CH == 0, "a chunk's pages lie in one 32-page window of the block table");
  static_assert(CHUNK_BYTES % 1024 == 0 && OFF_Q % 1024 == 0 && QHALF % 1024 == 0 && OFF_P % 1024 == 0,
                "128-byte swizzle atoms");
  static_assert(TM_S + NSB * CT <= TM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// An M = 64 product (and its operand A) keeps rows 16 q .. 16 q + 15 in lanes 0-15 of TMEM lane
// quarter q.

// 4-D tiled TMA load global -> shared, completion counted on `bar` in bytes (no cache hint).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}

// The same with an L2 cache policy.
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------- producer (warp 8)
// The loads that place an item (its work-list entry, block-table row) form a chain of dependent
// global reads.  The producer runs it ahead of the ring: while the chunks of item k are issued,
// the entry of item k + 2 and the block-table row of item k + 1 are in flight.
struct TcItemLoads {
  bool valid;
  WorkItem it;
  int kvh, rel0;
  int bt[4];  // block-table entries, one per lane for each 32-page window (items of up to 128 pages)
  bool mismatch;
};

template <typename C>
__device__ __forceinline__ void tc_produce(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                           const CUtensorMap& tmq, uint8_t* smem, uint64_t* bars, int4* meta,
                                           volatile int* abort_flag, int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int BS = C::BS;
  uint64_t* full = bars + C::B_FULL;
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* qfree = bars + C::B_QFREE;
  const int G = p.group, Hkv = p.num_kv_heads, T = p.qtok;
  const unsigned total = p.counters[1] * static_cast<unsigned>(Hkv);
  const uint64_t pol = policy_evict_first();
  // bytes of the query rows of one item: the box is G heads x (query tokens or members) rows, both halves
  const uint32_t qbytes = static_cast<uint32_t>(2 * G * p.qbox_rows * 128);
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
  auto entry = [&](unsigned w) -> WorkItem {
    return w < total ? p.items[w / Hkv] : WorkItem{0, 0, 0, 0, 0, 1, 0, 0};
  };
  // issue the block-table (and sequence-length) loads of item w (entry `it`); nothing waits here
  auto issue_loads = [&](unsigned w, const WorkItem& it, TcItemLoads& L) {
    L.valid = w < total;
    L.it = it;
    L.kvh = static_cast<int>(w % Hkv);
    L.bt[0] = L.bt[1] = L.bt[2] = L.bt[3] = 0;
    L.mismatch = false;
    L.rel0 = 0;
    if (!L.valid) return;
    const int members = (it.pm >> 16) & 0xff;
    const int npages = (it.tok1 - it.tok0 + BS - 1) / BS;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int pgi = lane + 32 * k;
      if (pgi < npages) {
        const int64_t col = it.tok0 / BS + pgi;
        L.bt[k] = p.block_tables[static_cast<int64_t>(it.seq) * p.max_blocks_per_seq + col];
        for (int m = 1; m < members; ++m)  // the members of a shared item must hold the same blocks
          L.mismatch |= p.block_tables[static_cast<int64_t>(it.seq + m) * p.max_blocks_per_seq + col] != L.bt[k];
      }
    }
    // key positions relative to the item's first query token, at position len - T + t0
    if (T > 1) L.rel0 = it.tok0 - (p.seq_lens[it.seq] - T + it.t0);
  };

  TcItemLoads cur, nxt;
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
    const int rows = members * it.tq;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) bad |= lane + 32 * k < npages && (cur.bt[k] < 0 || cur.bt[k] >= p.num_blocks);
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
    const int nch = (npages + C::CH - 1) / C::CH;
    for (int cc = 0; cc < nch; ++cc) {
      const int c = static_cast<int>(nchunks % C::NCH);
      if (!acquire(c)) {
        stop = true;
        break;
      }
      const int pg0 = cc * C::CH, npg = min(C::CH, npages - pg0);
      if (lane == 0) {
        const int ntok_last = min(BS, tok1 - (tok0 + (pg0 + npg - 1) * BS));
        const int flags = (cc == 0 ? F_FIRST : 0) | (cc == nch - 1 ? F_LAST : 0) | (bad ? F_BAD : 0) |
                          ((it.pm & WI_DIRECT) ? F_DIRECT : 0);
        meta[2 * c] = make_int4(it.seq, part, kvh | (npg << 8) | (rows << 16) | (flags << 24), cur.rel0 + pg0 * BS);
        meta[2 * c + 1] = make_int4(it.t0, ntok_last, static_cast<int>(qb), 0);
        if (bad)
          mbar_arrive(&full[c]);
        else
          mbar_arrive_expect_tx(&full[c], static_cast<uint32_t>(npg * 2 * C::VPAGE) + (cc == 0 ? qbytes : 0u));
        mbar_arrive(&bars[C::B_META + c]);  // roles that need only the meta go ahead
      }
      __syncwarp();  // the expected byte count is set before any copy can complete
      if (!bad) {
        // one box per lane: the K page / the V page, of page lane / 2 (a K page lands as [row
        // half][column block][8 rows], so the chunk's pages form the K operand with 8-row groups
        // 2048 bytes apart; a V page lands as [block][row])
        const int lp = lane >> 1, lk = lane & 1;
        // the chunk lies in one 32-page window (CH divides 32), so the window is warp-uniform
        const int win = pg0 >> 5;
        const int lphys = __shfl_sync(FULL, win == 0 ? cur.bt[0] : win == 1 ? cur.bt[1] : win == 2 ? cur.bt[2] : cur.bt[3],
                                      (pg0 + min(lp, C::CH - 1)) & 31);
        uint8_t* cb = smem + c * C::CHUNK_BYTES;
        if (lp < npg) {
          if (lk == 0)
            tma_load_4d_hint(cb + lp * C::KPAGE, &tmk, 0, 0, kvh * 2, lphys * (BS / 8), &full[c], pol);
          else
            tma_load_3d(cb + C::KC_BYTES + lp * C::VPAGE, &tmv, 0, lphys * BS, kvh * 2, &full[c], pol);
        }
        // the item's query rows with its first chunk: rows (query token or member) x G heads, one
        // box per 64-element half, landing as the K-major A operand
        if (cc == 0 && (lane == 16 || lane == 17))
          tma_load_4d(smem + C::OFF_Q + qb * C::QBUF + (lane - 16) * C::QHALF, &tmq, 0, lane - 16, kvh * G,
                      it.seq * T + it.t0, &full[c]);
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
        mbar_arrive(&bars[C::B_META + c]);
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

// ---------------------------------------------------------------- MMA issue (warps 9 and 10)
// Chunk meta as the MMA warps need it.
struct TcChunk {
  int c, npg, qb, item;
  bool end, poisoned, first, last;
};

// Warp 9: S(n) = Q . K(n)^T as soon as chunk n is in and its S buffer is free.  It also releases the
// query buffer once an item's last S is done, and takes part in releasing each chunk buffer (it
// has read the chunk's meta).
template <typename C>
__device__ __forceinline__ void tc_mma_s(uint8_t* smem, uint64_t* bars, const int4* meta, volatile int* abort_flag,
                                         uint32_t tm, int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int D = C::D;
  uint64_t* full = bars + C::B_FULL;
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* qfree = bars + C::B_QFREE;
  uint64_t* s_full = bars + C::B_SFULL;
  uint64_t* s_free = bars + C::B_SFREE;
  uint32_t ns = 0;  // S products issued
  bool item_bad = false, ok = true;
  int item_qb = 0;
  for (uint32_t k = 0;; ++k) {
    const int c = static_cast<int>(k % C::NCH);
    const bool ready = mbar_wait_bounded(&full[c], (k / C::NCH) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready && !*abort_flag)) {
      ok = false;
      break;
    }
    const int4 m0 = meta[2 * c], m1 = meta[2 * c + 1];
    const int flags = (m0.z >> 24) & 0xff;
    if (flags & F_END) break;
    if (flags & F_FIRST) {
      item_bad = (flags & F_BAD) != 0;
      item_qb = m1.z;
    }
    const bool last = (flags & F_LAST) != 0;
    if (!item_bad) {
      const uint32_t b = ns % C::NSB;
      if (ns >= C::NSB) {  // the softmax warps have read S(ns - NSB) out of this buffer
        const bool fr = mbar_wait_bounded(&s_free[b], ((ns / C::NSB) - 1) & 1u, kWaitLimit);
        if (!__all_sync(FULL, fr)) {
          ok = false;
          break;
        }
      }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + c * C::CHUNK_BYTES);
        const uint32_t qa = smem_u32(smem + C::OFF_Q + item_qb * C::QBUF);
#pragma unroll
        for (int k2 = 0; k2 < D / 16; ++k2) {
          const uint32_t a = qa + (k2 >> 2) * C::QHALF + (k2 & 3) * 32;
          const uint32_t bk = kb + (k2 >> 2) * 1024 + (k2 & 3) * 32;  // column block k2 / 4
          umma_ss(tm + C::TM_S + b * C::CT, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(bk, 16, 2048), C::IDESC_S,
                  k2 > 0);
        }
        umma_commit(&s_full[b]);
        if (last) umma_commit(&qfree[item_qb]);  // the query rows are read once the item's last S is done
      }
      __syncwarp();
      ++ns;
    } else if (last && lane == 0) {
      mbar_arrive(&qfree[item_qb]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[c]);  // this warp is done with the chunk's meta
  }
  if (!ok && lane == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
  // every product issued here completes before the tensor memory is released
  if (lane == 0) umma_commit(bars + C::B_FIN);
  __syncwarp();
  mbar_wait_bounded(bars + C::B_FIN, 0u, kWaitLimit);
}

// Warp 10: O_g += P(n) . V(n) once the softmax warps have written P(n), g the parity of n (the
// softmax group that took the chunk); its completion releases the P buffer and the chunk buffer.
// A group's first O product of an item overwrites its accumulator, once the item before has been
// read out of both.
template <typename C>
__device__ __forceinline__ void tc_mma_o(uint8_t* smem, uint64_t* bars, const int4* meta, volatile int* abort_flag,
                                         uint32_t tm, int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int D = C::D;
  uint64_t* meta_ready = bars + C::B_META;  // P full implies the chunk's copies landed (its S read them)
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* p_full = bars + C::B_PFULL;
  uint64_t* p_free = bars + C::B_PFREE;
  uint64_t* o_free = bars + C::B_OFREE;
  uint32_t np = 0;  // O products issued
  // items with O products (the others leave the accumulators alone), and the chunk's place in its item
  int items = -1, cc = 0;
  bool item_bad = false, ok = true;
  for (uint32_t k = 0;; ++k) {
    const int c = static_cast<int>(k % C::NCH);
    const bool ready = mbar_wait_bounded(&meta_ready[c], (k / C::NCH) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready && !*abort_flag)) {
      ok = false;
      break;
    }
    const int4 m0 = meta[2 * c];
    const int flags = (m0.z >> 24) & 0xff;
    if (flags & F_END) break;
    if (flags & F_FIRST) {
      item_bad = (flags & F_BAD) != 0;
      if (!item_bad) ++items;
      cc = 0;
    }
    const int npg = (m0.z >> 8) & 0xff;
    if (item_bad) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[c]);
      continue;
    }
    // the item's chunks alternate between the groups, so its first two open the two accumulators
    const bool opens = cc < 2;
    ++cc;
    const uint32_t pb = np & 1u, ob = np & 1u;
    bool good = mbar_wait_bounded(&p_full[pb], (np >> 1) & 1u, kWaitLimit);
    // the output of the item before (with O products: only those complete o_free, and an item's
    // output needs its own products, so o_free is never two items ahead) has been read out
    if (good && opens && items >= 1)
      good = mbar_wait_bounded(o_free, static_cast<uint32_t>(items - 1) & 1u, kWaitLimit);
    if (!__all_sync(FULL, good)) {
      ok = false;
      break;
    }
    if (lane == 0) {
      tc_fence_after();
      const uint32_t vb = smem_u32(smem + c * C::CHUNK_BYTES + C::KC_BYTES);
      const uint32_t pa = smem_u32(smem + C::OFF_P + pb * C::PBUF);
      for (int j = 0; j < npg; ++j) {
        const uint64_t a = smem_desc_sw128(pa + j * 32, 16, 1024);
        const uint64_t b = smem_desc_sw128(vb + j * C::VPAGE, C::BOX, 1024);
        umma_ss(tm + C::TM_O + ob * D, a, b, C::IDESC_O, (opens && j == 0) ? 0u : 1u);
      }
      umma_commit(&p_free[pb]);
      umma_commit(&empty[c]);  // the chunk buffer is free once these products are done
    }
    __syncwarp();
    ++np;
  }
  if (!ok && lane == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
  if (lane == 0) umma_commit(bars + C::B_FIN);
  __syncwarp();
  mbar_wait_bounded(bars + C::B_FIN, 0u, kWaitLimit);
}

// ---------------------------------------------------------------- kernel
template <typename KT, bool CAUSAL>
__global__ void __launch_bounds__(TcCfg<KT>::NTHREADS, 1)
    pa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const __grid_constant__ CUtensorMap tmq, const DecodeParams p) {
  using C = TcCfg<KT>;
  constexpr int D = C::D, CT = C::CT, HC = C::HC, M = C::M;
  // named barriers: 1 + q for the two softmax warps of lane quarter q; the softmax warps and the
  // MMA warps before the tensor memory is released
  constexpr int BAR_EXIT = 5;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);
  float2* xstate = reinterpret_cast<float2*>(smem + C::OFF_XCH);  // [item parity][group][M]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NBAR; ++s) {
      // S free and P full: one arrival per warp of the chunk's softmax group; O free: one per
      // softmax warp; a chunk buffer is free once the softmax warps and the S warp have read its
      // meta and the O warp has finished with it (or skipped it); the final drain: one commit per
      // MMA warp; item states: both warps of the quarter
      const bool grp = (s >= C::B_SFREE && s < C::B_SFREE + C::NSB) || (s >= C::B_PFULL && s < C::B_PFULL + 2);
      const bool all = s == C::B_OFREE;
      const bool empty = s >= C::B_EMPTY && s < C::B_EMPTY + C::NCH;
      const bool sums = s >= C::B_SUM && s < C::B_SUM + 8;
      mbar_init(&bars[s], grp ? C::NSM / 64 : all ? C::NSM / 32 : empty ? C::NSM / 32 + 2 : (s == C::B_FIN || sums) ? 2 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    prefetch_tensormap(&tmq);
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();  // the plan kernel's work list and counters are visible from here on

  if (warp == C::W_LOAD) {
    tc_produce<C>(p, tmk, tmv, tmq, smem, bars, meta, abort_flag, lane);
    return;
  }
  if (warp == C::W_S || warp == C::W_O) {
    if (warp == C::W_S)
      tc_mma_s<C>(smem, bars, meta, abort_flag, tm, lane);
    else
      tc_mma_o<C>(smem, bars, meta, abort_flag, tm, lane);
    tc_fence_before();
    bar_sync(BAR_EXIT, C::NSM + 64);
    return;
  }

  // ============================== softmax and output (warps 0-7) ==============================
  // Two groups of four warps take the S products in turn: group g = w / 4 the products whose index
  // has parity g, so that two chunks are in the softmax at once.  Warp w reads the 16 rows of lane
  // quarter q = w % 4 in the 16x256b shape: lane t holds rows 16 q + t / 4 and 16 q + t / 4 + 8 at
  // the chunk columns 8 j + 2 (t % 4), + 1 (j < 8).  Each group runs its own online softmax over its
  // chunks of the item, into its own O accumulator (O_g): its running maxima, raised lazily, its
  // row sums relative to them.  At the item's end the two warps of a quarter exchange their
  // groups' (maximum, sum) per row and each writes half of the head_dim columns of the combined
  // output, O = O_0 2^(m_0 - m) + O_1 2^(m_1 - m) with m the larger maximum.
  constexpr unsigned FULL = 0xffffffffu;
  constexpr float kNone = -1e30f;  // running maximum of a row with no score yet (finite: no NaN from -inf - -inf)
  constexpr int NJ = HC / 8;       // 8-column blocks of a chunk
  uint64_t* full = bars + C::B_FULL;
  uint64_t* meta_ready = bars + C::B_META;
  uint64_t* empty = bars + C::B_EMPTY;
  uint64_t* s_full = bars + C::B_SFULL;
  uint64_t* s_free = bars + C::B_SFREE;
  uint64_t* p_full = bars + C::B_PFULL;
  uint64_t* p_free = bars + C::B_PFREE;
  uint64_t* o_free = bars + C::B_OFREE;
  uint64_t* sum_bar = bars + C::B_SUM + 2 * (warp & 3);  // [item parity] of this quarter
  const int ct = threadIdx.x;
  const int quarter = warp & 3, grp = warp >> 2;
  const int gt = ct & 127;                                 // thread of the group
  const int rq = lane >> 2, cq = lane & 3;                 // row in the quarter's first eight, column pair
  const int row0 = quarter * 16 + rq, row1 = row0 + 8;     // this lane's two query rows
  const uint32_t tl = tm + (static_cast<uint32_t>(quarter * 32) << 16);  // the lane quarter (rows in lanes 0-15)
  const int G = p.group, Hq = p.num_q_heads, T = p.qtok, HV = T * Hq;
  const int rt0 = row0 / G, rt1 = row1 / G;  // the rows' query token (or member) in an item
  const float sl = p.scale_log2;
  uint32_t n = 0, ns = 0, np = 0;
  int items = -1;
  bool ok = true;
  float ml0 = kNone, ml1 = kNone;  // this group's running maxima of the item (log2 units)
  float l0 = 0.f, l1 = 0.f;        // this lane's part of the group's row sums, relative to them
  int ncol = 0, item_t0 = 0, first_np = 0, gk = 0;  // gk: this group's chunks of the item so far
  bool poisoned = false, busy = false;  // busy: the quarter holds at least one of the item's rows

  // completion of O product k (the P buffer it read is free again)
  auto wait_o = [&](uint32_t k) -> bool {
    const bool done = mbar_wait_bounded(&p_free[k & 1u], (k >> 1) & 1u, kWaitLimit);
    tc_fence_after();
    return done;
  };

  while (true) {
    const int c = static_cast<int>(n % C::NCH);
    const bool ready = mbar_wait_bounded(&meta_ready[c], (n / C::NCH) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready && !*abort_flag)) {
      ok = false;
      break;
    }
    const int4 mt0 = meta[2 * c], mt1 = meta[2 * c + 1];
    const int flags = (mt0.z >> 24) & 0xff;
    if (flags & F_END) break;
    const bool first = (flags & F_FIRST) != 0, last = (flags & F_LAST) != 0;
    if (first) {
      ++items;
      poisoned = (flags & F_BAD) != 0;
      ncol = ((mt0.z >> 16) & 0xff) * G;
      item_t0 = mt1.x;
      busy = quarter * 16 < ncol;
      ml0 = ml1 = kNone;
      l0 = l1 = 0.f;
      first_np = static_cast<int>(np);
      gk = 0;
    }
    const int npg = (mt0.z >> 8) & 0xff, ntok_last = mt1.y;
    uint8_t* cb = smem + c * C::CHUNK_BYTES;

    if (!poisoned) {
      const uint32_t k = ns++;  // this chunk's S product (np == k here)
      if ((k & 1u) == static_cast<uint32_t>(grp)) {
        bool good = true;
        if (ntok_last < C::BS) good = mbar_wait_bounded(&full[c], (n / C::NCH) & 1u, kWaitLimit);  // copies landed
        if (gt < CT && gt / C::BS == npg - 1 && (gt & (C::BS - 1)) >= ntok_last) {
          // V rows past the end of the item may hold anything (even NaN) and would meet zero
          // weights in the MMA: zero this token's row
          uint8_t* vrow = cb + C::KC_BYTES + (npg - 1) * C::VPAGE + (gt & (C::BS - 1)) * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) *reinterpret_cast<uint4*>(vrow + h * C::BOX + q * 16) = make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
        }
        const uint32_t b = k % C::NSB;
        good = mbar_wait_bounded(&s_full[b], (k / C::NSB) & 1u, kWaitLimit) && good;
        tc_fence_after();
        uint32_t sr[HC / 2];
        if (busy) {
          tmem_ld16x256<HC / 2>(tl + C::TM_S + b * CT, sr);
          tc_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[b]);

        // scores in log2 units, -inf where masked: tokens past the item's end; with several query
        // tokens, row r (query token r / G of the item) sees keys at relative positions <= r / G
        const int ntok = (npg - 1) * C::BS + ntok_last;
        auto jend_of = [&](int r, int rt) {
          return r < ncol ? (CAUSAL && T > 1 ? min(ntok, rt - mt0.w + 1) : ntok) : 0;
        };
        const int je0 = jend_of(row0, rt0), je1 = jend_of(row1, rt1);
        const int e0 = je0 - 2 * cq, e1 = je1 - 2 * cq;  // valid iff 8 j (+1) < e
        // the usual chunk: every row of the warp sees all its columns (no mask to apply)
        const bool whole = __all_sync(FULL, je0 >= CT && je1 >= CT);
        float x0 = -CUDART_INF_F, x1 = -CUDART_INF_F;
        auto chunk_max = [&](auto masked) {
          constexpr bool MK = decltype(masked)::value;
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            x0 = fmaxf(x0, fmaxf(!MK || 8 * j < e0 ? __uint_as_float(sr[4 * j]) : -CUDART_INF_F,
                                 !MK || 8 * j + 1 < e0 ? __uint_as_float(sr[4 * j + 1]) : -CUDART_INF_F));
            x1 = fmaxf(x1, fmaxf(!MK || 8 * j < e1 ? __uint_as_float(sr[4 * j + 2]) : -CUDART_INF_F,
                                 !MK || 8 * j + 1 < e1 ? __uint_as_float(sr[4 * j + 3]) : -CUDART_INF_F));
          }
        };
        if (busy) {
          if (whole)
            chunk_max(std::false_type{});
          else
            chunk_max(std::true_type{});
          x0 = fmaxf(x0, __shfl_xor_sync(FULL, x0, 1));
          x1 = fmaxf(x1, __shfl_xor_sync(FULL, x1, 1));
          x0 = fmaxf(x0, __shfl_xor_sync(FULL, x0, 2));
          x1 = fmaxf(x1, __shfl_xor_sync(FULL, x1, 2));
        }
        x0 *= sl;  // scale > 0 commutes with max
        x1 *= sl;
        // the group's maxima are raised only when a score exceeds them by more than the threshold
        const bool up0 = x0 > ml0 + kRescaleThreshold, up1 = x1 > ml1 + kRescaleThreshold;
        const float n0 = up0 ? x0 : ml0, n1 = up1 ? x1 : ml1;
        // O_g rows that already hold this item's products (those of the group's chunk k - 2) are
        // rescaled in tensor memory once that product is done (warp-wide ld / st: the warp votes)
        if (__any_sync(FULL, up0 || up1) && gk > 0) {
          const float a0 = up0 ? fast_exp2(ml0 - n0) : 1.f, a1 = up1 ? fast_exp2(ml1 - n1) : 1.f;
          good = wait_o(np - 2) && good;
#pragma unroll
          for (int h = 0; h < D / 32; ++h) {  // 32 columns of the O rows per pass
            uint32_t ov[16];
            tmem_ld16x256_x4(tl + C::TM_O + grp * D + h * 32, ov);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * ((i & 2) ? a1 : a0));
            tmem_st16x256_x4(tl + C::TM_O + grp * D + h * 32, ov);
          }
          tc_wait_st();
        }
        // the sums follow the maxima (0 from none)
        if (up0) l0 *= fast_exp2(ml0 - n0);
        if (up1) l1 *= fast_exp2(ml1 - n1);
        ml0 = n0;
        ml1 = n1;
        ++gk;
        // the weights the MMA sees; the sums are taken over the same rounded values
        uint32_t pk[2][NJ];
        auto chunk_weights = [&](auto masked) {
          constexpr bool MK = decltype(masked)::value;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float w0 = !MK || 8 * j < e0 ? fast_exp2(fmaf(__uint_as_float(sr[4 * j]), sl, -n0)) : 0.f;
            const float w1 = !MK || 8 * j + 1 < e0 ? fast_exp2(fmaf(__uint_as_float(sr[4 * j + 1]), sl, -n0)) : 0.f;
            const float w2 = !MK || 8 * j < e1 ? fast_exp2(fmaf(__uint_as_float(sr[4 * j + 2]), sl, -n1)) : 0.f;
            const float w3 = !MK || 8 * j + 1 < e1 ? fast_exp2(fmaf(__uint_as_float(sr[4 * j + 3]), sl, -n1)) : 0.f;
            pk[0][j] = pack2<KT>(w0, w1);
            pk[1][j] = pack2<KT>(w2, w3);
            const float2 r0 = unpack2<KT>(pk[0][j]), r1 = unpack2<KT>(pk[1][j]);
            s0 += r0.x + r0.y;
            s1 += r1.x + r1.y;
          }
          l0 += s0;
          l1 += s1;
        };
        if (busy) {
          if (whole)
            chunk_weights(std::false_type{});
          else
            chunk_weights(std::true_type{});
        } else {
#pragma unroll
          for (int j = 0; j < NJ; ++j) pk[0][j] = pk[1][j] = 0u;  // rows without the item's rows: zero weights
        }
        // this group's P buffer is free once O(k - 2) is done
        if (np >= 2) good = wait_o(np - 2) && good;
        if (!__all_sync(FULL, good)) {
          ok = false;
          break;
        }
        {  // K-major A operand: row r at r * 128, 16-byte chunk j (columns 8 j .. 8 j + 7) at
           // ((j ^ (r & 7)) << 4).  The warp's 16 rows x 64 columns are 16 matrices of 8 x 8 in the
           // fragment layout of pk (rows 0-7 in pk[0], 8-15 in pk[1]): four stmatrix.x4, the i-th
           // taking blocks 2 i and 2 i + 1; lane l gives row l % 8 of matrix l / 8 (rows + 8 for odd
           // l / 8, block + 1 for l / 8 >= 2).
          const int mrow = quarter * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          const uint32_t rbase = smem_u32(smem + C::OFF_P + (np & 1u) * C::PBUF) + mrow * 128;
          const int jsel = lane >> 4, rx = lane & 7;
#pragma unroll
          for (int i = 0; i < NJ / 2; ++i)
            stsm_x4(rbase + (((2 * i + jsel) ^ rx) << 4), pk[0][2 * i], pk[1][2 * i], pk[0][2 * i + 1], pk[1][2 * i + 1]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[np & 1u]);
      }
      ++np;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[c]);  // this warp is done with the chunk's meta and V rows

    if (last) {
      // output of the item: each warp writes half of the head_dim columns of its 16 rows
      const int nk = static_cast<int>(np) - first_np;  // the item's O products
      const bool bad = poisoned || nk == 0;
      bool good = true;
      if (!bad) good = wait_o(np - 1);  // all of them done (they complete in order)
      // the accumulators that hold the item's products: the group of its first chunk, and the
      // other one when it has two or more
      const bool even_me = (first_np & 1) == grp;  // this group took the item's chunks 0, 2, 4, ...
      const bool has_me = !bad && (nk >= 2 || even_me);
      const bool has_other = !bad && (nk >= 2 || !even_me);
      // this group's (maximum, sum) of the rows to the other warp of the quarter (one buffer per
      // item parity: every item, poisoned or not, ends with this exchange, so a buffer is
      // rewritten only after both warps have read it)
      l0 += __shfl_xor_sync(FULL, l0, 1);
      l1 += __shfl_xor_sync(FULL, l1, 1);
      l0 += __shfl_xor_sync(FULL, l0, 2);
      l1 += __shfl_xor_sync(FULL, l1, 2);
      const uint32_t ip = static_cast<uint32_t>(items) & 1u;
      float2* xs = xstate + ip * 2 * M;
      if (cq == 0) {
        xs[grp * M + row0] = make_float2(ml0, l0);
        xs[grp * M + row1] = make_float2(ml1, l1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sum_bar[ip]);
      good = mbar_wait_bounded(&sum_bar[ip], (static_cast<uint32_t>(items) >> 1) & 1u, kWaitLimit) && good;
      if (!__all_sync(FULL, good)) {
        ok = false;
        break;
      }
      const float2 ot0 = xs[(grp ^ 1) * M + row0], ot1 = xs[(grp ^ 1) * M + row1];
      // this warp's 64 columns of both accumulators, read at once (an accumulator without the
      // item's products is not read: its registers stay 0, tensor memory may hold anything there)
      uint32_t oe[2][16], oq[2][16];  // the even- and odd-place accumulators, 32 columns per pass
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int i = 0; i < 16; ++i) oe[h2][i] = oq[h2][i] = 0u;
      if (busy) {
        const uint32_t ce = tl + C::TM_O + (grp ^ (even_me ? 0 : 1)) * D + grp * 64;
        const uint32_t cqd = tl + C::TM_O + (grp ^ (even_me ? 1 : 0)) * D + grp * 64;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          if (even_me ? has_me : has_other) tmem_ld16x256_x4(ce + h2 * 32, oe[h2]);
          if (even_me ? has_other : has_me) tmem_ld16x256_x4(cqd + h2 * 32, oq[h2]);
        }
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      // the next item with O products may overwrite the accumulators (only such items complete
      // o_free: its phases then follow the O warp's count)
      if (!bad && lane == 0) mbar_arrive(o_free);
      if (busy) {
        const int seq = mt0.x, part = mt0.y & 0xffff, kvh = mt0.z & 0xff;
        const bool direct = (flags & F_DIRECT) != 0;
        int64_t ofs[2];
        // the factors of the accumulators of the item's even- and odd-place chunks, output scale
        // included: the two states are always combined in that order (which group takes which
        // chunks depends on the CTA's earlier items; the result does not)
        float fev[2], fod[2];
        bool live[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = i ? row1 : row0;
          const float mm = i ? ml1 : ml0, lm = i ? l1 : l0;
          const float2 ot = i ? ot1 : ot0;
          const float me = has_me ? mm : kNone, mo = has_other ? ot.x : kNone;
          const float mr = even_me ? fmaxf(me, mo) : fmaxf(mo, me);
          const float am = has_me ? fast_exp2(mm - mr) : 0.f, ao = has_other ? fast_exp2(ot.x - mr) : 0.f;
          const float ae = even_me ? am : ao, aod = even_me ? ao : am;
          const float lt = (even_me ? lm : ot.y) * ae + (even_me ? ot.y : lm) * aod;
          live[i] = r < ncol;
          const int mq = i ? rt1 : rt0, g = r - mq * G;
          const int mb = T > 1 ? 0 : mq, t = T > 1 ? item_t0 + mq : 0;
          const int vh = t * Hq + kvh * G + g;
          float f;
          if (direct) {
            ofs[i] = (static_cast<int64_t>(seq + mb) * HV + vh) * D;
            f = bad ? CUDART_NAN_F : p.v_scale / lt;
          } else {
            const int64_t pidx = static_cast<int64_t>(seq + mb) * p.max_parts + part;
            ofs[i] = (pidx * HV + vh) * D;
            f = bad ? CUDART_NAN_F : p.v_scale;
            if (live[i] && grp == 0 && cq == 0)
              __stcg(&p.part_ml[pidx * HV + vh], bad ? make_float2(0.f, CUDART_NAN_F) : make_float2(mr, lt));
          }
          fev[i] = ae * f;
          fod[i] = aod * f;
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int col0 = grp * 64 + h2 * 32;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (!live[i]) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int64_t e = ofs[i] + col0 + 8 * j + 2 * cq;
              const float a = __uint_as_float(oe[h2][4 * j + 2 * i]) * fev[i] +
                              __uint_as_float(oq[h2][4 * j + 2 * i]) * fod[i];
              const float b2 = __uint_as_float(oe[h2][4 * j + 2 * i + 1]) * fev[i] +
                               __uint_as_float(oq[h2][4 * j + 2 * i + 1]) * fod[i];
              if (!direct)
                __stcg(reinterpret_cast<float2*>(p.part_acc + e), make_float2(a, b2));
              else if (p.out_dtype == DT_F32)
                *reinterpret_cast<float2*>(static_cast<float*>(p.out) + e) = make_float2(a, b2);
              else
                *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + e) =
                    p.out_dtype == DT_BF16 ? pack2<__nv_bfloat16>(a, b2) : pack2<__half>(a, b2);
            }
          }
        }
      }
    }
    ++n;
  }
  if (!ok && lane == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
  tc_fence_before();
  bar_sync(BAR_EXIT, C::NSM + 64);  // the MMA warps have drained the tensor pipe
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, C::TM_COLS);
  }
}

}  // namespace pa
