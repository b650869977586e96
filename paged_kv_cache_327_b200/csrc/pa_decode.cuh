// pa_decode.cuh -- split-K paged decode attention for sm_100a.
//
// What is computed ("vLLM 深度解读", section 3, PagedAttention CUDA kernel): for each
// sequence i and query head hq, softmax over the sequence's tokens of
// scale * q[i,hq,:] . K_t, applied to V_t, where token t of sequence i sits in physical
// block block_tables[i][t / block_size] at position t % block_size, KV head hq / G.
//
// How (B200 design, not the page's one-CTA-per-(seq, head) scalar loop):
//  * plan kernel (one CTA): turns seq_lens (and prefix groups, if any) into a work list --
//    shared-prefix items first, then full 512-token partitions, then ragged tails -- zeroes
//    the work counter, and writes the rows of empty or invalid sequences;
//  * partition kernel: persistent, one CTA per SM, with NR rings (4, or 8 for an FP8 cache),
//    each fed by its own producer warp and drained by one consumer warp (two for items of more
//    than 8 query rows).  A work item is (sequence(s), token range, KV head), taken from an
//    atomic counter.  The producer resolves the item's block-table entries and streams its
//    pages into the ring of shared-memory slots: one TMA per 128-byte column block of the K
//    and V page (box = block_size rows x 128 B, 128-byte swizzle, L2 evict-first) plus bulk
//    copies of the item's query rows with the first page, counted on the slot's "full"
//    mbarrier; the consumers free the slot through its "empty" mbarrier.  Per page, all query
//    rows of the item (the G grouped heads, times the query tokens or the members of a shared
//    prefix) share one read of K and V:
//      S^T[tokens x rows] = K[tokens x D] . Q^T[D x rows]     (mma.sync m16n8k16, fp32 acc)
//      online softmax per row: exp2 of scale*log2(e)-scaled scores, with the running maximum
//      raised (and the accumulators rescaled) only when a score exceeds it by more than 2^8
//      -- the result is the same softmax, the rescale is rare; causal masking when the
//      sequence has several query tokens
//      O^T[D x rows] += V^T[D x tokens] . P^T[tokens x rows]  (P^T via movmatrix.trans)
//      l[rows]       += 1^T . P^T                             (one more MMA, no shuffles)
//    A sequence whose only item is one partition writes `out` directly.  Other items write
//    their (max, sum, unnormalised O) to the workspace and nothing else: no fence, atomic or
//    merge ever stalls a consumer's page stream;
//  * merge kernel: one warp per (sequence, query row) of a sequence with partial results
//    combines them with the log-sum-exp rescale, in a fixed order.
// The split depends only on seq_lens[i] (and the prefix groups) and each item is computed the
// same way whatever warp runs it, so results are deterministic; without prefix groups they are
// also batch-invariant.
#pragma once

#include <cuda_fp8.h>
#include <math_constants.h>

#include <type_traits>

#include "pa_ptx.cuh"

namespace pa {

enum : unsigned {
  DEV_OK = 0,
  DEV_BAD_BLOCK_ID = 1,
  DEV_BAD_SEQ_LEN = 2,
  DEV_BAD_SLOT = 3,
  DEV_BAD_PAIR = 4,
  DEV_TIMEOUT = 5,
  DEV_BAD_PREFIX = 6,
};

enum : int { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

// First data-dependent fault seen by any kernel of this library on this device.
__device__ unsigned int g_dev_error;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_dev_error, 0u, code); }

// polls of an mbarrier before a wait is declared dead
constexpr uint32_t kWaitLimit = 1u << 20;

// running maximum is raised only when a score exceeds it by more than this (log2 units)
constexpr float kRescaleThreshold = 8.0f;

// A work item: tokens [tok0, tok1) of sequence seq (and of the members - 1 sequences after it,
// which share those tokens' blocks), for every KV head, for the query tokens t0 .. t0 + tq - 1
// of the sequence (a sequence with more query tokens than one item holds is split into column
// groups); pm = part | members << 16 | WI_DIRECT.
struct __align__(16) WorkItem {
  int seq, tok0, tok1, pm;
  int t0, tq, pad0, pad1;
};
constexpr int WI_DIRECT = 1 << 30;  // the sequence's only item: write `out`, not a partial result

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int num_seqs, num_q_heads, num_kv_heads, group;
  int head_dim, block_size, max_blocks_per_seq, num_blocks;
  int partition_size, max_parts, out_dtype, qtok;  // qtok: query tokens per sequence (1 = decode)
  int qtok_item;     // query tokens of one item (qtok, or fewer: then several column groups)
  int qbox_rows;     // query rows per grouped head that the tensor-core kernel stages for an item
  // prefix groups, int32 [num_groups][3] = (first sequence, members, shared tokens): sequences
  // first .. first + members - 1 hold the same blocks for their first `shared` tokens
  const int32_t* groups;
  int num_groups, max_members;  // a shared item covers at most max_members sequences
  int long_partition;  // the longest item the partition kernel takes (a multiple of partition_size)
  int rings;           // page pipelines of the partition kernel (CTAs x rings per CTA)
  float scale_log2;  // scale * log2(e) (* k_scale for an FP8 cache)
  float v_scale;     // multiplies the output (FP8 cache); 1 otherwise
  // workspace views
  unsigned int* counters;  // [0] next work item, [1] number of work items
  WorkItem* items;         // [num_seqs * max_parts * column groups]
  int* seq_parts;          // [num_seqs]: partial results of the sequence (0: written directly, or no work)
  int* seq_shared;         // [num_seqs]: tokens shared through a valid prefix group (plan scratch)
  int* seq_sub;            // [num_seqs]: members of the shared items this sequence leads (plan scratch)
  float2* part_ml;         // [num_seqs * max_parts * qtok * num_q_heads]: (max in log2 units, sum)
  float* part_acc;         // [num_seqs * max_parts * qtok * num_q_heads * head_dim]
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
struct ScanSum {
  template <typename T>
  __device__ __forceinline__ T operator()(T a, T b) const { return a + b; }
};
struct ScanMax {
  template <typename T>
  __device__ __forceinline__ T operator()(T a, T b) const { return a > b ? a : b; }
};

template <typename T, typename Op>
__device__ __forceinline__ T warp_inclusive_scan(T v, Op op) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = op(n, v);
  }
  return v;
}

// Exclusive scan over the block (blockDim.x a multiple of 32, at most 1024) with an associative,
// commutative op whose identity is id; *total receives the reduction of all values.  A 64-bit T
// under ScanSum scans two 32-bit counts at once (low + high << 32).
template <typename T, typename Op>
__device__ T block_exclusive_scan(T v, T id, Op op, T* s_warp, T* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const T inc = warp_inclusive_scan(v, op);
  T exc = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) exc = id;
  if (lane == 31) s_warp[w] = inc;
  __syncthreads();
  if (w == 0) {
    const T x = lane < nw ? s_warp[lane] : id;
    const T xi = warp_inclusive_scan(x, op);
    T xe = __shfl_up_sync(0xffffffffu, xi, 1);
    if (lane == 0) xe = id;
    if (lane < nw) s_warp[lane] = xe;
    if (lane == 31) s_warp[32] = xi;
  }
  __syncthreads();
  const T r = op(s_warp[w], exc);
  *total = s_warp[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ long long pack2x32(int lo, int hi) {
  return static_cast<long long>(lo) + (static_cast<long long>(hi) << 32);
}
__device__ __forceinline__ int lo32(long long v) { return static_cast<int>(v & 0xffffffffll); }
__device__ __forceinline__ int hi32(long long v) { return static_cast<int>(v >> 32); }

constexpr int kPlanThreads = 1024;

// seq_parts values besides the partial-result count (0: the sequence's item writes `out`):
// rows the merge kernel fills, with zeros (an empty sequence) or NaN (an invalid length)
constexpr int kPartsEmpty = -1, kPartsInvalid = -2;

// Work list of one call.  Per sequence i of length L (valid: 0 <= L <= max_len and L = 0 or
// L >= qtok) with S shared tokens (0 outside a prefix group):
//   * shared items: a sequence that leads up to max_members members of a group gets one item
//     per partition of tokens [0, S), covering all those members;
//   * own items: tokens [S, L) in long partitions of Pb tokens, then partitions of Pm tokens,
//     then a ragged tail (Pb >= Pm >= P, all multiples of P, chosen below from the batch).
// The partial results of sequence i are numbered shared partitions first, then its own; a
// sequence with no shared tokens and one partition writes `out` directly.  Items are listed
// shared first (the widest), then long, then middle partitions, then tails, each kind in
// sequence order, so that the items that finish a launch are the shortest.
// Thread t plans the contiguous run of sequences [t * chunk, (t + 1) * chunk): every count
// is one block-wide scan, whatever the batch size.
__global__ void __launch_bounds__(kPlanThreads) pa_decode_plan_kernel(const DecodeParams p) {
  // the partition kernel may start its prologue now; it waits for this grid before
  // touching anything written here
  pdl_launch_dependents();
  __shared__ long long s_warp[33];
  const int N = p.num_seqs, P = p.partition_size, BS = p.block_size;
  const int max_len = p.max_blocks_per_seq * p.block_size;
  const int chunk = (N + blockDim.x - 1) / blockDim.x;
  const int lo = min(N, static_cast<int>(threadIdx.x) * chunk), hi = min(N, lo + chunk);
  auto valid_len = [&](int L) { return L >= 0 && L <= max_len && (L == 0 || L >= p.qtok); };

  if (p.num_groups > 0) {
    // A group is used if it is in range, its shared tokens are whole blocks that every member
    // holds, and no other group claims any of its sequences; otherwise it is reported and its
    // sequences decode alone.  Every group in range claims its members: claims start as a
    // difference array (+1 at first, -1 after the last member) whose prefix sum counts the
    // claims on each sequence; (1 + group index) is written at each group's first sequence, and a
    // prefix maximum of the positions that hold one finds, for a sequence claimed once, the
    // latest group start at or before it: the group that claims it.  A member rules its group out
    // if it is claimed more than once, its length is invalid or it holds fewer than the shared
    // tokens; an exclusive prefix count of such members gives each group's verdict in one
    // subtraction.  The verdicts are kept in the (not yet written) work list, one int per group
    // (num_groups <= N); seq_sub, seq_parts and seq_shared serve as scratch until their final
    // values are written.
    int* verdict = reinterpret_cast<int*>(p.items);
    int* claim = p.seq_sub;     // claims, then the claiming group of a sequence claimed once (or -1)
    int* cover = p.seq_parts;   // 1 + index of the group that starts at the sequence (0: none)
    int* badpre = p.seq_shared;
    const int* gr = p.groups;
    for (int i = threadIdx.x; i < N; i += blockDim.x) claim[i] = cover[i] = 0;
    __syncthreads();
    for (int g = threadIdx.x; g < p.num_groups; g += blockDim.x) {
      const int first = gr[3 * g], M = gr[3 * g + 1], S = gr[3 * g + 2];
      const bool ok = first >= 0 && M >= 1 && first <= N - M && S >= 0 && S % BS == 0;
      verdict[g] = ok;
      if (!ok) {
        record_error(DEV_BAD_PREFIX);
        continue;
      }
      atomicAdd(&claim[first], 1);
      if (first + M < N) atomicSub(&claim[first + M], 1);
      atomicMax(&cover[first], g + 1);
    }
    __syncthreads();
    int csum = 0, smax = 0;  // smax: 1 + the latest position holding a group start
    for (int i = lo; i < hi; ++i) {
      csum += claim[i];
      if (cover[i] > 0) smax = i + 1;
    }
    long long tot;
    int c = static_cast<int>(block_exclusive_scan<long long>(csum, 0, ScanSum{}, s_warp, &tot));
    int sp = static_cast<int>(block_exclusive_scan<long long>(smax, 0, ScanMax{}, s_warp, &tot));
    int nbad = 0;
    for (int i = lo; i < hi; ++i) {
      c += claim[i];
      if (cover[i] > 0) sp = i + 1;
      // a sequence claimed once lies in the group that starts last at or before it (cover is
      // only read here, so any thread may look up any start)
      const int g = c == 1 ? cover[sp - 1] - 1 : -1;
      bool bad = c > 1;
      if (g >= 0) {
        const int L = p.seq_lens[i];
        bad = !valid_len(L) || gr[3 * g + 2] > L;
      }
      claim[i] = g;
      badpre[i] = bad;
      nbad += bad;
    }
    int b = static_cast<int>(block_exclusive_scan<long long>(nbad, 0, ScanSum{}, s_warp, &tot));
    const int bad_total = static_cast<int>(tot);
    for (int i = lo; i < hi; ++i) {
      const int x = badpre[i];
      badpre[i] = b;
      b += x;
    }
    __syncthreads();
    for (int g = threadIdx.x; g < p.num_groups; g += blockDim.x) {
      if (!verdict[g]) continue;
      const int first = gr[3 * g], end = first + gr[3 * g + 1];
      if ((end < N ? badpre[end] : bad_total) != badpre[first]) {
        verdict[g] = 0;
        record_error(DEV_BAD_PREFIX);
      }
    }
    __syncthreads();
    // the sequences' shared tokens, and the members each leader of a shared pass covers
    for (int i = lo; i < hi; ++i) {
      int sh = 0, sub = 0;
      const int g = claim[i];
      if (g >= 0 && verdict[g]) {
        const int first = gr[3 * g], M = gr[3 * g + 1], S = gr[3 * g + 2];
        if (S > 0 && M > 1) {
          sh = S;
          const int k = i - first;
          if (k % p.max_members == 0) sub = min(p.max_members, M - k);
        }
      }
      p.seq_shared[i] = sh;
      p.seq_sub[i] = sub;
    }
    __syncthreads();  // the verdicts are dead from here on: the work list overwrites them
  }

  // column groups: the qtok query tokens of a sequence are split into items of qtok_item tokens
  const int Tc = p.qtok_item, ncg = (p.qtok + Tc - 1) / Tc;
  // Item lengths.  A longer item leaves fewer partial results for the merge and fewer item
  // starts and ends in the partition kernel, but the items that finish a launch set its tail.
  // Counted at P tokens, n items fall to each page pipeline; then shared items and long own
  // items take m P tokens (m up to long_partition / P) while at least 2 of them per pipeline
  // remain, and middle own items take m P tokens while at least 8 remain.  The choice is
  // block-uniform.
  int Ps = P, Pb = P, Pm = P;
  if (p.long_partition > P) {
    long long loc = 0, tot;  // shared items (low 32 bits) and own items (high 32 bits) at P
    for (int i = lo; i < hi; ++i) {
      const int L = p.seq_lens[i];
      if (!valid_len(L)) continue;
      const int S = p.num_groups > 0 ? p.seq_shared[i] : 0;
      if (p.num_groups > 0 && p.seq_sub[i] > 0) loc += (S + P - 1) / P;
      loc += static_cast<long long>((L - S + P - 1) / P * ncg) << 32;
    }
    (void)block_exclusive_scan<long long>(loc, 0, ScanSum{}, s_warp, &tot);
    const long long mmax = p.long_partition / P, hk = p.num_kv_heads, r = p.rings;
    const long long n_sh = (tot & 0xffffffffll) * hk, n_own = (tot >> 32) * hk;
    Ps = static_cast<int>(max(1ll, min(mmax, n_sh / (2 * r)))) * P;
    Pb = static_cast<int>(max(1ll, min(mmax, n_own / (2 * r)))) * P;
    Pm = static_cast<int>(max(1ll, min(mmax, n_own / (8 * r)))) * P;
  }
  struct Counts {
    int L, S, sub, ns, nb, nm, nt, nps;
  };
  auto counts = [&](int i) {
    Counts c{};
    c.L = p.seq_lens[i];
    if (!valid_len(c.L)) return c;
    c.S = p.num_groups > 0 ? p.seq_shared[i] : 0;
    c.sub = p.num_groups > 0 ? p.seq_sub[i] : 0;
    c.nps = (c.S + Ps - 1) / Ps;
    c.ns = c.sub > 0 ? c.nps : 0;
    const int own = c.L - c.S;
    c.nb = Pb > Pm ? own / Pb : 0;
    c.nm = (own - c.nb * Pb) / Pm;
    c.nt = ((own - c.nb * Pb) % Pm) ? 1 : 0;
    return c;
  };

  int loc_s = 0, loc_b = 0, loc_m = 0, loc_t = 0;
  for (int i = lo; i < hi; ++i) {
    const Counts c = counts(i);
    loc_s += c.ns;
    loc_b += c.nb * ncg;
    loc_m += c.nm * ncg;
    loc_t += c.nt * ncg;
  }
  long long t_bm, t_ts;
  const long long o_bm = block_exclusive_scan<long long>(pack2x32(loc_b, loc_m), 0, ScanSum{}, s_warp, &t_bm);
  const long long o_ts = block_exclusive_scan<long long>(pack2x32(loc_t, loc_s), 0, ScanSum{}, s_warp, &t_ts);
  int ob = lo32(o_bm), om = hi32(o_bm), ot = lo32(o_ts), os = hi32(o_ts);
  const int n_long = lo32(t_bm), n_mid = hi32(t_bm), n_tail = lo32(t_ts), n_shared = hi32(t_ts);
  // own items follow the shared ones: long, then middle, then tails
  ob += n_shared;
  om += n_shared + n_long;
  ot += n_shared + n_long + n_mid;
  for (int i = lo; i < hi; ++i) {
    const Counts c = counts(i);
    const bool valid = valid_len(c.L);
    if (!valid) record_error(DEV_BAD_SEQ_LEN);
    const int parts = c.nps + c.nb + c.nm + c.nt;
    const bool direct = c.S == 0 && parts == 1;
    p.seq_parts[i] = !valid ? kPartsInvalid : c.L == 0 ? kPartsEmpty : direct ? 0 : parts;
    const int dflag = direct ? WI_DIRECT : 0;
    // shared items have one query token (prefix groups are single-token decode)
    for (int k = 0; k < c.ns; ++k)
      p.items[os++] = WorkItem{i, k * Ps, min(c.S, (k + 1) * Ps), k | (c.sub << 16), 0, 1, 0, 0};
    // own partitions: [tok0, tok1) as partial result `part`, one item per column group
    auto own_item = [&](int& o, int tok0, int tok1, int part) {
      for (int j = 0; j < ncg; ++j)
        p.items[o++] = WorkItem{i, tok0, tok1, part | (1 << 16) | dflag, j * Tc, min(Tc, p.qtok - j * Tc), 0, 0};
    };
    int tok = c.S, part = c.nps;
    for (int k = 0; k < c.nb; ++k, tok += Pb) own_item(ob, tok, tok + Pb, part++);
    for (int k = 0; k < c.nm; ++k, tok += Pm) own_item(om, tok, tok + Pm, part++);
    if (c.nt) own_item(ot, tok, c.L, part);
  }
  if (threadIdx.x == 0) {
    p.counters[0] = 0;
    p.counters[1] = static_cast<unsigned>(n_shared + n_long + n_mid + n_tail);
  }
}

// ------------------------------------------------------------------------------ partition kernel
// Tag of a KV cache holding FP8 E4M3 codes (one byte per element).  Its tiles are turned into
// f16 in registers, so its tensor-core work runs in f16; the query is then split into two f16
// parts (hi + lo) to keep its precision.
struct fp8e4m3 {};

template <typename KT>
struct KvTraits {
  using mma_t = KT;
  static constexpr int bytes = 2;
  static constexpr bool fp8 = false;
};
template <>
struct KvTraits<fp8e4m3> {
  using mma_t = __half;
  static constexpr int bytes = 1;
  static constexpr bool fp8 = true;
};

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_float<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// four E4M3 codes (byte 0 first) -> f16 pairs (bytes 0, 1) and (bytes 2, 3), exact (every E4M3
// value is an f16 value); the two halves of the word are converted in place, with no shift
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t v, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(v));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}


// NT: 8-column MMA tiles per consumer warp; PAIR: two consumer warps share each ring, the
// second taking the item's query rows after the first's 8 * NT (for items of up to 32 rows:
// twice the warps hide the latency of the longer per-page work); CAUSAL: the kernel can run
// several query tokens per sequence (causal masking compiled in); NR: rings per CTA, each with
// its own producer warp (8 rings put two independent consumers on every scheduler, for the
// FP8 cache whose consumers convert every tile).
template <int BS, int D, typename KT, typename QT, int NT, bool PAIR, bool CAUSAL, int NR = 4>
struct DecodeCfg {
  static constexpr bool FP8 = KvTraits<KT>::fp8;
  static constexpr int HALVES = D * KvTraits<KT>::bytes / 128;  // 128-byte column blocks of a row
  static constexpr int BOX_BYTES = BS * 128;            // one TMA box: BS rows x 128 bytes
  static constexpr int PAGE_BYTES = BOX_BYTES * HALVES; // one KV head of one block
  static constexpr int QE = sizeof(QT);
  // an fp32 query is split into hi + lo parts of the operand type; a 16-bit query over an FP8
  // cache is converted to f16 once (exact for |q| in [2^-14, 65504])
  static constexpr bool QSPLIT = std::is_same<QT, float>::value;
  static constexpr bool QCONV = FP8 && !QSPLIT;
  static constexpr int CONS = PAIR ? 2 : 1;             // consumer warps per ring
  static constexpr int COLS = 8 * NT * CONS;            // query rows per item (MMA N dimension)
  static constexpr int QBUF_BYTES = ((COLS * D * QE + 1023) / 1024) * 1024;  // one item's query rows
  // query buffers per ring: the producer fills item k's while items k - QN + 1 .. k - 1 are in
  // flight, so it can run ahead across short items
  static constexpr int QN = (PAIR || NR > 4) ? 2 : 4;
  static constexpr int SLOT_BYTES = 2 * PAGE_BYTES;     // K page then V page
  static constexpr int NC = NR;                         // rings, one producer warp each
  static constexpr int NCONS = NC * CONS;               // consumer warps: ring = warp % NC
  static constexpr int NWARP = NCONS + NC;
  // registers per thread: at launch (65536 / threads, a multiple of 8), and -- with more than 8
  // warps -- after setmaxnreg moves the producers' share to the consumers
  static constexpr bool SPLIT = NWARP > 8;
  static constexpr int REG_LAUNCH = SPLIT ? (65536 / (NWARP * 32)) & ~7 : 255;
  static constexpr int REG_PRODUCER = 56;
  static constexpr int REG_CONSUMER = SPLIT ? ((NWARP * REG_LAUNCH - NC * REG_PRODUCER) / NCONS) & ~7 : 255;
  static_assert(!SPLIT || NC * 32 * REG_PRODUCER + NCONS * 32 * REG_CONSUMER <= NWARP * 32 * REG_LAUNCH,
                "register split exceeds the launch allocation");
  static_assert(!SPLIT || (NC % 4 == 0 && NCONS % 4 == 0), "setmaxnreg acts on whole warpgroups");
  static constexpr int SMEM_BUDGET = 200 * 1024;
  static constexpr int NSLOT_FIT = (SMEM_BUDGET / NC - QN * QBUF_BYTES) / SLOT_BYTES;
  static constexpr int NSLOT = NSLOT_FIT > 8 ? 8 : (NSLOT_FIT < 2 ? 2 : NSLOT_FIT);
  static constexpr int RING_BYTES = NC * (NSLOT * SLOT_BYTES + QN * QBUF_BYTES);
  static constexpr int NBAR = (2 * NSLOT + QN + 1) & ~1;     // full + empty per slot, qfree per buffer (+pad)
  static constexpr int BAR_BYTES = NC * NBAR * 8;
  static constexpr int META_BYTES = NC * NSLOT * 32;    // two int4 per slot
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + META_BYTES + 16 * NC;
  static constexpr int MT = BS / 16;    // 16-token MMA tiles per page
  static constexpr int KS = D / 16;     // 16-wide steps over head_dim
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(BS == 16 || BS == 32, "block_size");
  static_assert(HALVES >= 1, "an FP8 row must fill a 128-byte box (head_dim 128)");
  static_assert((NT == 1 && !PAIR && !CAUSAL) || (!FP8 && !QSPLIT), "wide or causal items: 16-bit cache and query");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// byte offset, inside a page, of the 16-byte chunk holding (row t, columns d0..d0+7)
// under the TMA 128-byte swizzle (chunk index XOR row mod 8 within each 1024-byte atom)
template <int BOX_BYTES>
__device__ __forceinline__ uint32_t swz(int t, int d0) {
  return (d0 >> 6) * BOX_BYTES + t * 128 + ((((d0 & 63) >> 3) ^ (t & 7)) << 4);
}

// slot metadata, two int4 per slot: [0] x = seq, y = part | page << 16,
// z = kvh | ntok << 8 | rows << 16 | flags << 24 (rows: members x query tokens of the item),
// w = position of the page's first token relative to the item's first query token;
// [1] x = the item's first query token t0
constexpr int F_FIRST = 1, F_LAST = 2, F_BAD = 4, F_END = 8, F_DIRECT = 16;

// The producer warp of one ring: takes work items from the shared counter and streams their pages
// (K and V of one KV head, by TMA) and query rows (bulk copies) into the ring's slots, with each
// slot's metadata; ends the stream with an F_END slot.  C gives the slot geometry.
template <class C, int BS, int D>
__device__ __forceinline__ void produce(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                        uint8_t* ring, uint8_t* qbufs, uint64_t* full, uint64_t* empty,
                                        uint64_t* qfree, int4* meta, volatile int* abort_flag, int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  const int G = p.group, Hkv = p.num_kv_heads, Hq = p.num_q_heads, T = p.qtok;
  const unsigned total = p.counters[1] * static_cast<unsigned>(Hkv);
  const uint64_t pol = policy_evict_first();
  uint32_t n = 0;      // pages issued into this ring
  uint32_t items = 0;  // items started (the query buffer is refilled once per item)
  bool stop = false;
  auto acquire_slot = [&](int slot) -> bool {  // wait until the consumer freed `slot`
    if (n < C::NSLOT) return true;
    const bool ok = mbar_wait_bounded(&empty[slot], ((n / C::NSLOT) - 1) & 1u, kWaitLimit);
    return __all_sync(FULL, ok) && !*abort_flag;
  };
  while (!stop) {
    unsigned w = 0;
    if (lane == 0) w = atomicAdd(&p.counters[0], 1u);
    w = __shfl_sync(FULL, w, 0);
    if (w >= total) break;
    const WorkItem it = p.items[w / Hkv];
    const int kvh = static_cast<int>(w % Hkv);
    const int part = it.pm & 0xffff, members = (it.pm >> 16) & 0xff;
    const int tok0 = it.tok0, tok1 = it.tok1;
    const int npages = (tok1 - tok0 + BS - 1) / BS;
    const int t0 = it.t0, tq = it.tq;
    const int rows = members * tq;  // (member, query token) pairs of the item: G query rows each
    // key positions relative to the item's first query token, at position len - T + t0
    // (causal masking of several query tokens)
    const int rel0 = T > 1 ? tok0 - (p.seq_lens[it.seq] - T + t0) : 0;
    // the item's block-table entries, one per lane for each 32-page window (items of up to 128
    // pages; all of them are checked before the first page goes out)
    bool bad = false, mismatch = false;
    auto entry = [&](int pgi) -> int {
      int v = 0;
      if (pgi < npages) {
        const int64_t col = tok0 / BS + pgi;
        v = p.block_tables[static_cast<int64_t>(it.seq) * p.max_blocks_per_seq + col];
        bad |= v < 0 || v >= p.num_blocks;
        // the members of a shared item must hold the same blocks
        for (int m = 1; m < members; ++m)
          mismatch |= p.block_tables[static_cast<int64_t>(it.seq + m) * p.max_blocks_per_seq + col] != v;
      }
      return v;
    };
    const int bt0 = entry(lane), bt1 = entry(lane + 32), bt2 = entry(lane + 64), bt3 = entry(lane + 96);
    bad = __any_sync(FULL, bad);
    mismatch = __any_sync(FULL, mismatch);
    if (lane == 0) {
      if (bad) record_error(DEV_BAD_BLOCK_ID);
      if (mismatch) record_error(DEV_BAD_PREFIX);
    }
    bad |= mismatch;
    const uint32_t qb = items % C::QN;
    if (items >= C::QN) {  // the consumers have taken the query rows of item `items - QN`
      const bool ok = mbar_wait_bounded(&qfree[qb], ((items / C::QN) - 1) & 1u, kWaitLimit);
      if (!__all_sync(FULL, ok) || *abort_flag) {
        stop = true;
        break;
      }
    }
    for (int pg = 0; pg < npages; ++pg) {
      const int win = pg >> 5;  // warp-uniform
      const int phys = __shfl_sync(FULL, win == 0 ? bt0 : win == 1 ? bt1 : win == 2 ? bt2 : bt3, pg & 31);
      const int slot = static_cast<int>(n % C::NSLOT);
      if (!acquire_slot(slot)) {
        stop = true;
        break;
      }
      const bool first = pg == 0;
      if (lane == 0) {
        uint8_t* sb = ring + slot * C::SLOT_BYTES;
        const int ntok = min(BS, tok1 - (tok0 + pg * BS));
        const int flags = (first ? F_FIRST : 0) | (pg == npages - 1 ? F_LAST : 0) | (bad ? F_BAD : 0) |
                          ((it.pm & WI_DIRECT) ? F_DIRECT : 0);
        meta[2 * slot] = make_int4(it.seq, part | (pg << 16), kvh | (ntok << 8) | (rows << 16) | (flags << 24),
                                   rel0 + pg * BS);
        meta[2 * slot + 1] = make_int4(t0, 0, 0, 0);
        if (bad) {
          mbar_arrive(&full[slot]);
        } else {
          const uint32_t qbytes = first ? static_cast<uint32_t>(rows * G * D * C::QE) : 0u;
          mbar_arrive_expect_tx(&full[slot], 2 * C::PAGE_BYTES + qbytes);
          if constexpr (C::HALVES == 2) {  // one box per page: both column blocks of the KV head row
            tma_load_3d(sb, &tmk, 0, phys * BS, kvh * 2, &full[slot], pol);
            tma_load_3d(sb + C::PAGE_BYTES, &tmv, 0, phys * BS, kvh * 2, &full[slot], pol);
          } else {
            tma_load_3d(sb, &tmk, 0, kvh, phys * BS, &full[slot], pol);
            tma_load_3d(sb + C::PAGE_BYTES, &tmv, 0, kvh, phys * BS, &full[slot], pol);
          }
        }
      }
      if (first && !bad) {
        __syncwarp();  // the expected byte count is set before any copy can complete
        if (lane < rows) {  // query rows of (member, token) lane: G contiguous heads
          const int m = lane / tq, t = t0 + lane - m * tq;
          bulk_load(qbufs + qb * C::QBUF_BYTES + lane * G * D * C::QE,
                    static_cast<const uint8_t*>(p.q) +
                        ((static_cast<int64_t>(it.seq + m) * T + t) * Hq + kvh * G) * D * C::QE,
                    static_cast<uint32_t>(G * D * C::QE), &full[slot]);
        }
      }
      ++n;
    }
    ++items;
  }
  if (!stop) {  // tell the consumer there is no more work
    const int slot = static_cast<int>(n % C::NSLOT);
    if (acquire_slot(slot)) {
      if (lane == 0) {
        meta[2 * slot] = make_int4(0, 0, F_END << 24, 0);
        mbar_arrive(&full[slot]);
      }
    } else {
      stop = true;
    }
  }
  if (stop) {
    if (lane == 0) record_error(DEV_TIMEOUT);
    // copies this warp issued may still be landing: wait for them before the CTA exits
    for (uint32_t k = n > C::NSLOT ? n - C::NSLOT : 0; k < n; ++k)
      mbar_wait_bounded(&full[k % C::NSLOT], (k / C::NSLOT) & 1u, kWaitLimit);
  }
}

// The query rows ("columns") of one work item are (member m, query token t, head g) for
// m < members, t < qtok, g < G, in that order: column c = (m * qtok + t) * G + g.  A plain decode
// has one member and one query token; multi-token attention has qtok > 1 (query token t sits at
// position len - qtok + t and attends causally); a shared-prefix item has members > 1 (the
// sequences seq .. seq + members - 1 share the item's tokens).
template <int BS, int D, typename KT, typename QT, int NT, bool PAIR, bool CAUSAL, int NR>
__global__ void __launch_bounds__(DecodeCfg<BS, D, KT, QT, NT, PAIR, CAUSAL, NR>::NWARP * 32, 1)
    pa_decode_partition_kernel(const __grid_constant__ CUtensorMap tmk,
                               const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
  using C = DecodeCfg<BS, D, KT, QT, NT, PAIR, CAUSAL, NR>;
  using MA = typename KvTraits<KT>::mma_t;  // element type of the tensor-core operands
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = warp % C::NC;  // ring of this warp (its consumers and producer share a scheduler)
  uint8_t* ring = smem + c * (C::NSLOT * C::SLOT_BYTES + C::QN * C::QBUF_BYTES);
  uint8_t* qbufs = ring + C::NSLOT * C::SLOT_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES) + c * C::NBAR;
  uint64_t* empty = full + C::NSLOT;
  uint64_t* qfree = empty + C::NSLOT;
  int4* meta = reinterpret_cast<int4*>(smem + C::RING_BYTES + C::BAR_BYTES) + 2 * c * C::NSLOT;
  volatile int* flags_base = reinterpret_cast<volatile int*>(smem + C::RING_BYTES + C::BAR_BYTES + C::META_BYTES);
  volatile int* abort_flag = flags_base + 4 * c;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NC; ++i) {
      uint64_t* b = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES) + i * C::NBAR;
      // full: the producer's arrival (+ bytes); empty and qfree: one arrival per consumer warp
      for (int s = 0; s < 2 * C::NSLOT + C::QN; ++s) mbar_init(&b[s], s < C::NSLOT ? 1 : C::CONS);
      flags_base[4 * i] = 0;
    }
    fence_mbar_init();
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  __syncthreads();
  pdl_wait();  // the plan kernel's work list and counters are visible from here on

  const int G = p.group, Hq = p.num_q_heads, T = p.qtok;

  if (warp >= C::NCONS) {
    // ============================== producer ==============================
    if constexpr (C::SPLIT) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::REG_PRODUCER));
    produce<C, BS, D>(p, tmk, tmv, ring, qbufs, full, empty, qfree, meta, abort_flag, lane);
    return;
  }

  // ============================== consumer ==============================
  if constexpr (C::SPLIT) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::REG_CONSUMER));
  const int col0 = (warp / C::NC) * NT * 8;  // first query row (column) of this consumer
  const int lr = lane & 7, lm = lane >> 3;  // ldmatrix: row inside an 8x8 matrix, matrix index
  const int r0 = lane >> 2, c2 = (lane & 3) * 2;
  // per-lane swizzled offsets of the ldmatrix rows (the same in every slot and 16-row tile).
  // Step k adds 2k to the 16-byte chunk index, an even number, so under the XOR swizzle its
  // offset is the step-0 offset XOR (k mod 4) << 5, plus the 128-byte column block k / 4.
  const uint32_t koff0 = swz<C::BOX_BYTES>(lr + ((lm & 1) << 3), (lm >> 1) << 3);
  const uint32_t voff0 = swz<C::BOX_BYTES>(lr + ((lm >> 1) << 3), (lm & 1) << 3);
  auto koff = [&](int k) { return (koff0 ^ ((k & 3) << 5)) + (k >> 2) * C::BOX_BYTES; };
  auto voff = [&](int k) { return (voff0 ^ ((k & 3) << 5)) + (k >> 2) * C::BOX_BYTES; };
  const float sl = p.scale_log2;
  const uint32_t ones = pack2<MA>(1.f, 1.f);
  // FP8 tiles: per-lane offsets of the K rows for ldmatrix (row lr + 8 (lm & 1), 16-byte chunk
  // 2 kb + (lm >> 1)) and the swizzle terms of the V rows 2c (+8) and 2c+1 (+8) a lane reads
  uint32_t koff8[C::FP8 ? C::KS / 2 : 1];
  int vx0 = 0, vx1 = 0;
  if constexpr (C::FP8) {
#pragma unroll
    for (int kq = 0; kq < C::KS / 2; ++kq) {
      const int t = lr + ((lm & 1) << 3);
      koff8[kq] = t * 128 + ((((2 * kq + (lm >> 1)) ^ (t & 7))) << 4);
    }
    vx0 = c2 & 7;
    vx1 = (c2 + 1) & 7;
  }

  float mu[NT][2];  // running maxima (log2 units) of columns nt * 8 + c2, + 1
  float acc[C::KS][NT][4] = {};
  float lacc[NT][4] = {};
  uint32_t qf[C::KS][NT][2];
  uint32_t ql[C::QSPLIT ? C::KS : 1][2];
  (void)ql;
  bool poisoned = false;
  int ncol = G;       // query rows of the current item
  int item_t0 = 0;    // its first query token

  // query rows of the item from its buffer qbuf; rows >= ncol are zero
  auto load_q = [&](const uint8_t* qbuf) {
    if constexpr (!C::QSPLIT && !C::QCONV) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int k2 = 0; k2 < C::KS; k2 += 2) {
          const int d0 = (k2 + (lm >> 1)) * 16 + ((lm & 1) << 3);
          ldsm_x4(smem_u32(qbuf + ((col0 + nt * 8 + lr) * D + d0) * 2), qf[k2][nt][0], qf[k2][nt][1],
                  qf[k2 + 1][nt][0], qf[k2 + 1][nt][1]);
        }
        if (col0 + nt * 8 + r0 >= ncol) {
#pragma unroll
          for (int k = 0; k < C::KS; ++k) qf[k][nt][0] = qf[k][nt][1] = 0u;
        }
      }
    } else {
      const QT* qv = reinterpret_cast<const QT*>(qbuf);
      const bool live = r0 < ncol;
#pragma unroll
      for (int kk = 0; kk < C::KS; ++kk) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // FP8 tiles are unpacked as 4 consecutive columns 16 kk + 4c .. +3 per lane
          // (pairs h = 0, 1); the query takes the same order.  Otherwise the usual
          // m16n8k16 columns 16 kk + 2c (+1) and + 8.
          const int d = C::FP8 ? kk * 16 + 2 * c2 + 2 * h : kk * 16 + h * 8 + c2;
          const float x0 = live ? to_float(qv[r0 * D + d]) : 0.f, x1 = live ? to_float(qv[r0 * D + d + 1]) : 0.f;
          const uint32_t hi = pack2<MA>(x0, x1);
          qf[kk][0][h] = hi;
          if constexpr (C::QSPLIT) {
            const float2 hf = unpack2<MA>(hi);
            ql[kk][h] = pack2<MA>(x0 - hf.x, x1 - hf.y);
          }
        }
      }
    }
  };

  // One page: S^T = K . Q^T, online-softmax update, O^T += V^T . P^T.  The softmax state is
  // updated once per chunk of MC 16-token tiles: the whole page for items of up to 16 query
  // rows, each tile on its own for wider items (their scores would not fit in registers).
  // na: the number NA of 8-column tiles that hold the current item's query rows (NT, or 1 for an
  // item of at most 8 rows -- items of one call differ in width when shared items cover several
  // sequences); the tiles past NA are skipped.  The choice is made once per page, so the tile
  // loops stay unrolled and branch-free.
  auto page_math = [&](const uint8_t* sb, int ntok, int rel, auto na) {
    constexpr int NA = decltype(na)::value;
    auto on = [](int nt) { return nt < NA; };
    const uint32_t kb = smem_u32(sb), vb = kb + C::PAGE_BYTES;
    constexpr int MC = NA > 1 ? 1 : C::MT;
#pragma unroll
    for (int m0 = 0; m0 < C::MT; m0 += MC) {
      float s[MC][NT][4];
#pragma unroll
      for (int mi = 0; mi < MC; ++mi) {
        const int mt = m0 + mi;
        float sa[NT][4] = {}, sb2[NT][4] = {};
        if constexpr (C::FP8) {
          // one ldmatrix.x4 holds 32 columns of 16 rows: lane gets 4 codes of row r0 (r0 + 8)
#pragma unroll
          for (int kq = 0; kq < C::KS / 2; ++kq) {
            uint32_t r[4];
            ldsm_x4(kb + mt * 2048 + koff8[kq], r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int kk = 2 * kq + h;
              uint32_t a0, a1, a2, a3;
              e4m3x4_to_f16x2x2(r[2 * h], a0, a2);
              e4m3x4_to_f16x2x2(r[2 * h + 1], a1, a3);
              if constexpr (C::QSPLIT) {
                Mma<MA>::run(sa[0], a0, a1, a2, a3, qf[kk][0][0], qf[kk][0][1]);
                Mma<MA>::run(sb2[0], a0, a1, a2, a3, ql[kk][0], ql[kk][1]);
              } else {
                Mma<MA>::run(h ? sb2[0] : sa[0], a0, a1, a2, a3, qf[kk][0][0], qf[kk][0][1]);
              }
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < C::KS; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kb + mt * 2048 + koff(kk), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (!on(nt)) continue;
              if constexpr (C::QSPLIT) {
                Mma<MA>::run(sa[nt], a0, a1, a2, a3, qf[kk][nt][0], qf[kk][nt][1]);
                Mma<MA>::run(sb2[nt], a0, a1, a2, a3, ql[kk][0], ql[kk][1]);
              } else if (kk & 1) {
                Mma<MA>::run(sb2[nt], a0, a1, a2, a3, qf[kk][nt][0], qf[kk][nt][1]);
              } else {
                Mma<MA>::run(sa[nt], a0, a1, a2, a3, qf[kk][nt][0], qf[kk][nt][1]);
              }
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[mi][nt][e] = sa[nt][e] + sb2[nt][e];
      }
      if (ntok < BS) {  // tokens past the end of the partition do not take part
#pragma unroll
        for (int mi = 0; mi < MC; ++mi)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if ((m0 + mi) * 16 + r0 + 8 * h >= ntok) s[mi][nt][2 * h] = s[mi][nt][2 * h + 1] = -CUDART_INF_F;
      }
      if (CAUSAL && T > 1 && rel + BS > 1) {
        // causal: query token t sees keys up to its own position (rel: the page's first key
        // relative to query token 0)
#pragma unroll
        for (int mi = 0; mi < MC; ++mi)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = col0 + nt * 8 + c2 + (e & 1);
              const int t = col / G;  // the item's query token (one member when T > 1)
              if (rel + (m0 + mi) * 16 + r0 + 8 * (e >> 1) > t) s[mi][nt][e] = -CUDART_INF_F;
            }
      }
      // raw (unscaled) maxima of this lane's entries; scale > 0 commutes with max
      float x[NT][2];
      bool raise = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        x[nt][0] = x[nt][1] = -CUDART_INF_F;
#pragma unroll
        for (int mi = 0; mi < MC; ++mi) {
          x[nt][0] = fmaxf(x[nt][0], fmaxf(s[mi][nt][0], s[mi][nt][2]));
          x[nt][1] = fmaxf(x[nt][1], fmaxf(s[mi][nt][1], s[mi][nt][3]));
        }
        if (on(nt))
          raise |= x[nt][0] * sl > mu[nt][0] + kRescaleThreshold || x[nt][1] * sl > mu[nt][1] + kRescaleThreshold;
      }
      if (__any_sync(FULL, raise)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (!on(nt)) continue;
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            x[nt][0] = fmaxf(x[nt][0], __shfl_xor_sync(FULL, x[nt][0], o));
            x[nt][1] = fmaxf(x[nt][1], __shfl_xor_sync(FULL, x[nt][1], o));
          }
          const float n0 = fmaxf(mu[nt][0], x[nt][0] * sl), n1 = fmaxf(mu[nt][1], x[nt][1] * sl);
          // a column that has seen only masked scores keeps -inf; its weights stay 0
          const float al0 = n0 == -CUDART_INF_F ? 1.f : fast_exp2(mu[nt][0] - n0);
          const float al1 = n1 == -CUDART_INF_F ? 1.f : fast_exp2(mu[nt][1] - n1);
          mu[nt][0] = n0;
          mu[nt][1] = n1;
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            acc[dt][nt][0] *= al0;
            acc[dt][nt][1] *= al1;
            acc[dt][nt][2] *= al0;
            acc[dt][nt][3] *= al1;
          }
          lacc[nt][0] *= al0;
          lacc[nt][1] *= al1;
          lacc[nt][2] *= al0;
          lacc[nt][3] *= al1;
        }
      }
#pragma unroll
      for (int mi = 0; mi < MC; ++mi) {
        const int mt = m0 + mi;
        uint32_t b0[NT], b1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          b0[nt] = b1[nt] = 0u;
          if (!on(nt)) continue;
          // a column with no visible key yet (mu = -inf) gets weight 0, not 2^(-inf + inf)
          const float u0 = mu[nt][0] == -CUDART_INF_F ? 0.f : mu[nt][0];
          const float u1 = mu[nt][1] == -CUDART_INF_F ? 0.f : mu[nt][1];
          const uint32_t plo =
              pack2<MA>(fast_exp2(fmaf(s[mi][nt][0], sl, -u0)), fast_exp2(fmaf(s[mi][nt][1], sl, -u1)));
          const uint32_t phi =
              pack2<MA>(fast_exp2(fmaf(s[mi][nt][2], sl, -u0)), fast_exp2(fmaf(s[mi][nt][3], sl, -u1)));
          b0[nt] = movmatrix_t(plo);
          b1[nt] = movmatrix_t(phi);
          Mma<MA>::run(lacc[nt], ones, ones, ones, ones, b0[nt], b1[nt]);  // row sums of the weights the MMA sees
        }
        if constexpr (C::FP8) {
          // V^T tiles (16 columns x 16 tokens) from the codes, two MMA steps per load: in step
          // pair sp a lane reads one 32-bit word -- columns d .. d + 3 with
          // d = 32 sp + 16 (r0 >> 2) + 4 (r0 & 3) -- of tokens 2c, 2c+1, 2c+8, 2c+9, and pairs
          // the tokens up by byte permutation: step 2 sp takes columns d, d + 1 (accumulator
          // rows r0, r0 + 8), step 2 sp + 1 columns d + 2, d + 3.
          const int tk = mt * 16 + c2;
          const uint32_t rowa = vb + (mt * 16 + c2) * 128 + 4 * (r0 & 3);  // tokens 2c (+8)
          const uint32_t rowb = rowa + 128;                                  // tokens 2c+1 (+9)
          auto v_tiles = [&](uint32_t mlo, uint32_t mhi, auto masked) {
#pragma unroll
            for (int sp = 0; sp < C::KS / 2; ++sp) {
              const int chunk = 2 * sp + (r0 >> 2);  // 16-byte chunk of the row holding the word
              const uint32_t w0 = lds_u32(rowa + ((chunk ^ vx0) << 4));
              const uint32_t w1 = lds_u32(rowb + ((chunk ^ vx1) << 4));
              const uint32_t w2 = lds_u32(rowa + 8 * 128 + ((chunk ^ vx0) << 4));
              const uint32_t w3 = lds_u32(rowb + 8 * 128 + ((chunk ^ vx1) << 4));
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint32_t sel = h ? 0x7362u : 0x5140u;  // columns d, d+1 or d+2, d+3
                uint32_t a0, a1, a2, a3;
                e4m3x4_to_f16x2x2(__byte_perm(w0, w1, sel), a0, a1);
                e4m3x4_to_f16x2x2(__byte_perm(w2, w3, sel), a2, a3);
                if constexpr (decltype(masked)::value) {
                  a0 &= mlo;
                  a1 &= mlo;
                  a2 &= mhi;
                  a3 &= mhi;
                }
                Mma<MA>::run(acc[2 * sp + h][0], a0, a1, a2, a3, b0[0], b1[0]);
              }
            }
          };
          if (ntok >= (mt + 1) * 16) {
            v_tiles(FULL, FULL, std::false_type{});
          } else {
            const uint32_t mlo = (tk < ntok ? 0x0000ffffu : 0u) | (tk + 1 < ntok ? 0xffff0000u : 0u);
            const uint32_t mhi = (tk + 8 < ntok ? 0x0000ffffu : 0u) | (tk + 9 < ntok ? 0xffff0000u : 0u);
            v_tiles(mlo, mhi, std::true_type{});
          }
        } else if (ntok >= (mt + 1) * 16) {
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vb + mt * 2048 + voff(dt), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              if (on(nt)) Mma<MA>::run(acc[dt][nt], a0, a1, a2, a3, b0[nt], b1[nt]);
          }
        } else {
          // V rows past the end may hold anything (even NaN): zero them, 0 * NaN would poison
          const int tk = mt * 16 + c2;
          const uint32_t mlo = (tk < ntok ? 0x0000ffffu : 0u) | (tk + 1 < ntok ? 0xffff0000u : 0u);
          const uint32_t mhi = (tk + 8 < ntok ? 0x0000ffffu : 0u) | (tk + 9 < ntok ? 0xffff0000u : 0u);
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vb + mt * 2048 + voff(dt), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              if (on(nt)) Mma<MA>::run(acc[dt][nt], a0 & mlo, a1 & mlo, a2 & mhi, a3 & mhi, b0[nt], b1[nt]);
          }
        }
      }
    }  // chunk of MC tiles
  };

  // Write the item's result.  Column col = (m * T + t) * G + g is query head kvh * G + g of
  // query token t of sequence seq + m; its "virtual head" (T query tokens x Hq heads) is
  // t * Hq + kvh * G + g.
  auto finalize = [&](int seq, int part, int kvh, bool direct) {
    const float nan = CUDART_NAN_F;
    // accumulator rows r0 and r0 + 8 of tile dt are columns d = vcol(dt) and d + dd
    const int dd = C::FP8 ? 1 : 8;
    auto vcol = [&](int dt) {
      return C::FP8 ? 32 * (dt >> 1) + 16 * (r0 >> 2) + 4 * (r0 & 3) + 2 * (dt & 1) : dt * 16 + r0;
    };
    const float vs = p.v_scale;
    const int HV = T * Hq;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = col0 + nt * 8 + c2 + j;
        if (col >= ncol) continue;
        const int g = col % G, mt_ = col / G;
        // several query tokens: one member, token t0 + mt_; otherwise member mt_, token 0
        const int m = T > 1 ? 0 : mt_, t = T > 1 ? item_t0 + mt_ : 0;
        const int vh = t * Hq + kvh * G + g;
        const float l = lacc[nt][j];  // every row of the ones-MMA holds the column sums
        if (direct) {
          const float inv = poisoned ? nan : vs / l;
          const int64_t o = (static_cast<int64_t>(seq + m) * HV + vh) * D;
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            const int d = vcol(dt);
            store_out(p.out, o + d, acc[dt][nt][j] * inv, p.out_dtype);
            store_out(p.out, o + d + dd, acc[dt][nt][2 + j] * inv, p.out_dtype);
          }
        } else {
          const int64_t pidx = static_cast<int64_t>(seq + m) * p.max_parts + part;
          float* pa = p.part_acc + (pidx * HV + vh) * D;
#pragma unroll
          for (int dt = 0; dt < C::KS; ++dt) {
            const int d = vcol(dt);
            __stcg(pa + d, poisoned ? nan : acc[dt][nt][j] * vs);
            __stcg(pa + d + dd, poisoned ? nan : acc[dt][nt][2 + j] * vs);
          }
          if (r0 == 0)
            __stcg(&p.part_ml[pidx * HV + vh], poisoned ? make_float2(0.f, nan) : make_float2(mu[nt][j], l));
        }
      }
    }
  };

  uint32_t n = 0;
  uint32_t citems = 0;  // items started by this consumer (selects the query buffer)
  bool ok = true;
  while (true) {
    const int slot = static_cast<int>(n % C::NSLOT);
    // every lane waits (acquire); the vote keeps the warp together if a wait gives up
    const bool ready = mbar_wait_bounded(&full[slot], (n / C::NSLOT) & 1u, kWaitLimit);
    if (!__all_sync(FULL, ready)) {
      ok = false;
      break;
    }
    const int4 mt = meta[2 * slot];
    const int kvh = mt.z & 0xff, ntok = (mt.z >> 8) & 0xff, flags = (mt.z >> 24) & 0xff;
    if (flags & F_END) break;
    const int part = mt.y & 0xffff;
    const uint8_t* sb = ring + slot * C::SLOT_BYTES;
    if (flags & F_FIRST) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mu[nt][0] = mu[nt][1] = -CUDART_INF_F;
        lacc[nt][0] = lacc[nt][1] = lacc[nt][2] = lacc[nt][3] = 0.f;
#pragma unroll
        for (int dt = 0; dt < C::KS; ++dt) acc[dt][nt][0] = acc[dt][nt][1] = acc[dt][nt][2] = acc[dt][nt][3] = 0.f;
      }
      poisoned = (flags & F_BAD) != 0;
      ncol = ((mt.z >> 16) & 0xff) * G;  // (members x query tokens of the item) x grouped heads
      item_t0 = meta[2 * slot + 1].x;
      const uint32_t qb = citems % C::QN;
      if (!poisoned) load_q(qbufs + qb * C::QBUF_BYTES);
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfree[qb]);  // the buffer may take a later item's rows
      ++citems;
    }
    const int mycols = ncol - col0;  // query rows of the item in this consumer's tiles
    if (!poisoned && mycols > 0) {
      if (NT > 1 && mycols <= 8)
        page_math(sb, ntok, mt.w, std::integral_constant<int, 1>{});
      else
        page_math(sb, ntok, mt.w, std::integral_constant<int, NT>{});
    }
    __syncwarp();  // every lane is done reading the slot before it is handed back
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (flags & F_LAST) finalize(mt.x, part, kvh, (flags & F_DIRECT) != 0);
    ++n;
  }
  if (!ok && lane == 0) {
    record_error(DEV_TIMEOUT);
    *abort_flag = 1;
  }
}

// ------------------------------------------------------------------------------ self-test
// A wait that nothing completes: the bounded wait gives up after `polls` polls, records
// DEV_TIMEOUT and the kernel returns (the failure path of every wait in this library).
__global__ void __launch_bounds__(32) pa_selftest_wait_kernel(uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = mbar_wait_bounded(&bar, 0, polls);  // phase 0 never completes
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) record_error(DEV_TIMEOUT);
}

// ------------------------------------------------------------------------------ merge
// One warp per (sequence, virtual head = query token x query head) of a sequence whose items
// wrote partial results (shared partitions first, then its own):
// out = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k, M = max_k m_k, taken in one pass over the
// partitions in order: a running maximum, with the numerator and denominator relative to it
// rescaled whenever a later partition raises it (the same quotient).  The loads of kMergeBatch
// partitions are in flight at once; each lane holds head_dim / 32 consecutive columns.
constexpr int kMergeWarps = 8;
constexpr int kMergeBatch = 4;

__device__ __forceinline__ float neg_inf() { return -CUDART_INF_F; }

template <int V>  // columns per lane
struct MergeRow {
  float m, den, num[V];
  __device__ __forceinline__ MergeRow() : m(neg_inf()), den(0.f) {
#pragma unroll
    for (int j = 0; j < V; ++j) num[j] = 0.f;
  }
  // partition k: (maximum, sum, this lane's columns of the unnormalised output).  A partition in
  // which the row saw no key is (-inf, 0, 0) and adds nothing; a poisoned one carries NaN.
  __device__ __forceinline__ void add(float mk, float lk, const float (&a)[V]) {
    if (mk == neg_inf()) return;
    if (mk > m) {
      const float r = fast_exp2(m - mk);  // 0 while nothing has been added (m = -inf)
      den *= r;
#pragma unroll
      for (int j = 0; j < V; ++j) num[j] *= r;
      m = mk;
    }
    const float w = fast_exp2(mk - m);
    den += w * lk;
#pragma unroll
    for (int j = 0; j < V; ++j) num[j] += w * a[j];
  }
};

template <int V>
__device__ __forceinline__ void merge_row(const DecodeParams& p, int64_t base, int np, int64_t vrow, int HV,
                                          int64_t o, int lane) {
  using VT = typename std::conditional<V == 4, float4, float2>::type;
  constexpr int D = 32 * V;
  MergeRow<V> acc;
  for (int k0 = 0; k0 < np; k0 += kMergeBatch) {
    float2 ml[kMergeBatch];
    float a[kMergeBatch][V];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
      if (k0 + u < np) {
        const int64_t row = (base + k0 + u) * HV + vrow;
        ml[u] = __ldcg(&p.part_ml[row]);
        const VT x = __ldcg(reinterpret_cast<const VT*>(p.part_acc + row * D) + lane);
        const float* xf = reinterpret_cast<const float*>(&x);
#pragma unroll
        for (int j = 0; j < V; ++j) a[u][j] = xf[j];
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u)
      if (k0 + u < np) acc.add(ml[u].x, ml[u].y, a[u]);
  }
  const float inv = 1.f / acc.den;
#pragma unroll
  for (int j = 0; j < V; ++j) store_out(p.out, o + lane * V + j, acc.num[j] * inv, p.out_dtype);
}

__global__ void __launch_bounds__(kMergeWarps * 32, 4) pa_decode_merge_kernel(const DecodeParams p) {
  pdl_wait();  // the partition kernel's partial results are visible from here on
  const int lane = threadIdx.x & 31;
  const int64_t pair = static_cast<int64_t>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  const int Hq = p.qtok * p.num_q_heads, D = p.head_dim;
  if (pair >= static_cast<int64_t>(p.num_seqs) * Hq) return;
  const int seq = static_cast<int>(pair / Hq), hq = static_cast<int>(pair % Hq);
  const int np = p.seq_parts[seq];  // the plan's count of the sequence's partial results
  const int64_t o = (static_cast<int64_t>(seq) * Hq + hq) * D;
  if (np < 0) {  // no work item: the row is zero (empty sequence) or NaN (invalid length)
    const float v = np == kPartsEmpty ? 0.f : CUDART_NAN_F;
    for (int d = lane; d < D; d += 32) store_out(p.out, o + d, v, p.out_dtype);
    return;
  }
  if (np == 0) return;  // written directly by the sequence's only item
  const int64_t base = static_cast<int64_t>(seq) * p.max_parts;
  if (D == 128)
    merge_row<4>(p, base, np, hq, Hq, o, lane);
  else
    merge_row<2>(p, base, np, hq, Hq, o, lane);
}

}  // namespace pa
