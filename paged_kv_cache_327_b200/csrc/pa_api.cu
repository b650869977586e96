// pa_api.cu -- the C ABI of libpa.so (declared in include/pa.h): host-side validation,
// workspace layout, TMA descriptor encoding and kernel launches.  Every step of the
// computation runs in the CUDA kernels of pa_decode.cuh / pa_cache.cuh; there is no CPU
// fallback.  No call allocates device memory: the library's only device memory is static (the
// error word and the fixed scratch buffer of pa_decode_static_workspace).
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <unordered_set>

#include "pa.h"
#include "pa_cache.cuh"
#include "pa_decode_tc.cuh"

namespace {

constexpr int kDefaultPartition = 512;
constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int elem_bytes(int dt) { return dt == PA_F32 ? 4 : dt == PA_FP8_E4M3 ? 1 : 2; }

struct WsLayout {
  size_t counters, seq_parts, seq_shared, seq_sub, items, part_ml, part_acc, total;
};

// Partitions a sequence of up to max_len tokens can produce: its own ceil(max_len / P), plus one
// with prefix groups, where a shared prefix may end inside a partition (shared and own tokens
// are partitioned apart).  The workspace size covers both.
int64_t max_parts_for(int64_t max_len, int P, bool groups = true) {
  return std::max<int64_t>(1, (max_len + P - 1) / P + (groups ? 1 : 0));
}

// Query rows one work item holds per KV head on the warp-MMA kernels: 32 with head_dim 128, 8 with
// head_dim 64; the tensor-core kernel holds up to kTcMaxRows.
int max_item_rows(int head_dim) { return head_dim == 128 ? 32 : 8; }
constexpr int kTcMaxRows = 64;

// Work items of one partition of one sequence, bounded from num_q_heads (= query tokens x query
// heads) alone.  A split item holds floor(max_rows / G) * G >= 28 rows with head_dim 128 and
// >= 5 with head_dim 64 (G <= 8), so ceil(num_q_heads / 16), resp. ceil(num_q_heads / 4), items
// cover every column group; an unsplit partition has one item.
int64_t items_per_partition_bound(int64_t num_q_heads, int64_t head_dim) {
  const int64_t min_rows = head_dim == 128 ? 16 : 4;
  return std::max<int64_t>(1, (num_q_heads + min_rows - 1) / min_rows);
}

// num_q_heads: query heads x query tokens.  Items: one per (sequence, partition, column group).
WsLayout ws_layout(int64_t num_seqs, int64_t num_q_heads, int64_t head_dim, int64_t max_parts) {
  WsLayout L{};
  size_t o = 0;
  L.counters = o;
  o += 256;
  L.seq_parts = o;
  o += align256(static_cast<size_t>(num_seqs) * sizeof(int));
  L.seq_shared = o;
  o += align256(static_cast<size_t>(num_seqs) * sizeof(int));
  L.seq_sub = o;
  o += align256(static_cast<size_t>(num_seqs) * sizeof(int));
  L.items = o;
  o += align256(static_cast<size_t>(num_seqs * max_parts * items_per_partition_bound(num_q_heads, head_dim)) *
                sizeof(pa::WorkItem));
  L.part_ml = o;
  o += align256(static_cast<size_t>(num_seqs * max_parts * num_q_heads) * sizeof(float2));
  L.part_acc = o;
  o += align256(static_cast<size_t>(num_seqs * max_parts * num_q_heads * head_dim) * sizeof(float));
  L.total = o;
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Per-device launch facts, looked up once.
struct DeviceInfo {
  int sm_count = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(int* dev, DeviceInfo** info) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[*dev];
  if (d.sm_count == 0 && cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
    return PA_ERR_CUDA;
  *info = &d;
  return PA_OK;
}

// KV cache [num_blocks, block_size, num_kv_heads, head_dim] seen as a 3-D tensor of 128-byte
// column blocks (head_dim * elem / 128 of them per KV head), 128-byte swizzle:
//  * per block: dims (128 bytes of a row, column blocks, num_blocks * block_size rows); one box =
//    block_size rows of one column block, coordinates (0, column block, row);
//  * whole rows (two_blocks, a KV head row of two column blocks): dims (128 bytes, rows, column
//    blocks) with strides (row pitch, 128 bytes) -- the outer stride below the middle one; one box
//    = block_size rows of both column blocks of a KV head, landing as [block][row][128 bytes], the
//    layout two per-block boxes give; coordinates (0, row, column block).
int encode_kv_map(CUtensorMap* map, const void* base, int kv_dtype, int64_t num_blocks, int block_size,
                  int num_kv_heads, int head_dim, bool two_blocks = false) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return PA_ERR_CUDA;
  const int es = elem_bytes(kv_dtype);
  const cuuint64_t inner = 128 / es;
  const cuuint64_t nblk = static_cast<cuuint64_t>(head_dim * es / 128) * num_kv_heads;
  const cuuint64_t rows = static_cast<cuuint64_t>(num_blocks) * block_size;
  const cuuint64_t pitch = static_cast<cuuint64_t>(num_kv_heads) * head_dim * es;
  const cuuint64_t dims_b[3] = {inner, nblk, rows}, dims_r[3] = {inner, rows, nblk};
  const cuuint64_t strides_b[2] = {128, pitch}, strides_r[2] = {pitch, 128};
  const cuuint32_t box_b[3] = {static_cast<cuuint32_t>(inner), 1, static_cast<cuuint32_t>(block_size)};
  const cuuint32_t box_r[3] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(block_size), 2};
  const cuuint64_t* dims = two_blocks ? dims_r : dims_b;
  const cuuint64_t* strides = two_blocks ? strides_r : strides_b;
  const cuuint32_t* box = two_blocks ? box_r : box_b;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = kv_dtype == PA_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : kv_dtype == PA_F16  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// A 16-bit K cache with head_dim 128 for the tensor-core kernel, seen as a 4-D tensor (64 elements,
// 8 rows, column blocks of 64 elements of every KV head, groups of 8 rows): one box = the page of
// one KV head (2 column blocks x 16 rows), landing as [row half][column block][8 rows][128 bytes]
// with the 128-byte swizzle.  Consecutive pages of a chunk then hold each column block's 8-row
// groups 2048 bytes apart: the K-major operand of a 64-token S product, one box per page.
int encode_k_tc_map(CUtensorMap* map, const void* base, int kv_dtype, int64_t num_blocks, int block_size,
                    int num_kv_heads) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return PA_ERR_CUDA;
  const cuuint64_t pitch = static_cast<cuuint64_t>(num_kv_heads) * 256;  // bytes of a token row
  const cuuint64_t groups = static_cast<cuuint64_t>(num_blocks) * block_size / 8;
  const cuuint64_t dims[4] = {64, 8, static_cast<cuuint64_t>(num_kv_heads) * 2, groups};
  const cuuint64_t strides[3] = {pitch, 128, 8 * pitch};
  const cuuint32_t box[4] = {64, 8, 2, static_cast<cuuint32_t>(block_size / 8)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = kv_dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// The query [num_seqs * qtok rows, num_q_heads, head_dim] (16-bit) seen as a 4-D tensor (64
// elements, 2 halves of head_dim, heads, rows); one box = the 64-element half of `box_rows` rows of
// G consecutive heads, 128-byte swizzle: the K-major A operand of the tensor-core kernel.
int encode_q_map(CUtensorMap* map, const void* q, int q_dtype, int64_t rows, int num_q_heads, int G, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return PA_ERR_CUDA;
  const cuuint64_t dims[4] = {64, 2, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[3] = {128, 256, static_cast<cuuint64_t>(num_q_heads) * 256};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = q_dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = enc(map, dt, 4, const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

template <int BS, int D, typename KT, typename QT, int NT, bool PAIR, bool CAUSAL, int NR>
int launch_partition(const pa::DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                     int64_t max_items, int dev, DeviceInfo* info, cudaStream_t stream) {
  using C = pa::DecodeCfg<BS, D, KT, QT, NT, PAIR, CAUSAL, NR>;
  auto kern = pa::pa_decode_partition_kernel<BS, D, KT, QT, NT, PAIR, CAUSAL, NR>;
  static std::atomic<bool> smem_set[kMaxDevices];  // per instantiation and device
  if (!smem_set[dev].load(std::memory_order_acquire)) {
    if (C::SPLIT) {
      // the warps' setmaxnreg split must fit the registers the block is launched with, or the
      // consumers' increase would wait for ever: never launch such a build
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PA_ERR_CUDA;
      if (fa.numRegs < C::REG_LAUNCH) return PA_ERR_UNSUPPORTED;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return PA_ERR_CUDA;
    smem_set[dev].store(true, std::memory_order_release);
  }
  int64_t ctas = (max_items + C::NWARP - 1) / C::NWARP;
  if (ctas > info->sm_count) ctas = info->sm_count;
  if (ctas < 1) ctas = 1;
  // programmatic dependent launch: the prologue overlaps the plan kernel, which the
  // partition kernel waits for (griddepcontrol.wait) before reading anything
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(C::NWARP * 32);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tmk, tmv, p) != cudaSuccess) return PA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The tensor-core kernel for wide items (block size 16, head_dim 128, 16-bit cache and query).
// kernel for items of more than 8 query rows (PA_OPT_WIDE_KERNEL)
std::atomic<int> g_wide_kernel{PA_WIDE_AUTO};
// how the calls cut sequences into work items (PA_OPT_ITEM_SPLIT)
std::atomic<int> g_item_split{PA_SPLIT_ADAPTIVE};

template <typename KT>
int launch_tc(const pa::DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tmq,
              int64_t max_items, int dev, DeviceInfo* info, cudaStream_t stream) {
  using C = pa::TcCfg<KT>;
  auto kern = pa::pa_decode_tc_kernel<KT, true>;
  static std::atomic<bool> smem_set[kMaxDevices];
  if (!smem_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return PA_ERR_CUDA;
    smem_set[dev].store(true, std::memory_order_release);
  }
  int64_t ctas = max_items;  // one ring (and one CTA) per SM
  if (ctas > info->sm_count) ctas = info->sm_count;
  if (ctas < 1) ctas = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(C::NTHREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tmk, tmv, tmq, p) != cudaSuccess) return PA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Kernel instantiation for (block_size, head_dim, KV dtype, query dtype, query rows per item,
// several query tokens): single-token items of up to 8 query rows run on every dtype pair with one
// consumer warp per ring; multi-token items of up to 8 rows on a 16-bit cache with a query of the
// same type; wider items (several query tokens, or the members of a shared prefix) on a 16-bit
// cache with a query of the same type, head_dim 128, with two consumer warps per ring of 1 or 2
// eight-row tiles.
template <int BS, int D>
int dispatch_kv(const pa::DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap* tmq,
                const CUtensorMap* tmk_blocks, int64_t max_items, int dev, DeviceInfo* info, int kv_dtype,
                int q_dtype, int cols, cudaStream_t stream) {
  const bool qf32 = q_dtype == PA_F32;
  const int nt = (cols + 7) / 8;
  // one instantiation: KV element type K, query type Q, tiles per consumer N, paired, causal;
  // an FP8 cache runs 8 rings per CTA
  auto run = [&](auto k, auto q, auto n, auto pair, auto causal) {
    using K = decltype(k);
    using Q = decltype(q);
    constexpr int NR = std::is_same<K, pa::fp8e4m3>::value ? 8 : 4;
    return launch_partition<BS, D, K, Q, decltype(n)::value, decltype(pair)::value, decltype(causal)::value, NR>(
        p, tmk, tmv, max_items, dev, info, stream);
  };
  using bf16 = __nv_bfloat16;
  using f16 = __half;
  using One = std::integral_constant<int, 1>;
  using Two = std::integral_constant<int, 2>;
  using Yes = std::true_type;
  using No = std::false_type;
  if (nt == 1 && p.qtok > 1) {
    if (kv_dtype == PA_BF16 && q_dtype == PA_BF16) return run(bf16{}, bf16{}, One{}, No{}, Yes{});
    if (kv_dtype == PA_F16 && q_dtype == PA_F16) return run(f16{}, f16{}, One{}, No{}, Yes{});
    return PA_ERR_UNSUPPORTED;
  }
  if (nt > 1) {
    if constexpr (D == 128 && BS == 16) {  // 5th-generation tensor-core kernel, when chosen
      if (tmq) {
        if (kv_dtype == PA_BF16 && q_dtype == PA_BF16)
          return launch_tc<bf16>(p, *tmk_blocks, tmv, *tmq, max_items, dev, info, stream);
        if (kv_dtype == PA_F16 && q_dtype == PA_F16)
          return launch_tc<f16>(p, *tmk_blocks, tmv, *tmq, max_items, dev, info, stream);
      }
    }
    if constexpr (D == 128) {
      if (kv_dtype == PA_BF16 && q_dtype == PA_BF16)
        return nt == 2 ? run(bf16{}, bf16{}, One{}, Yes{}, Yes{}) : run(bf16{}, bf16{}, Two{}, Yes{}, Yes{});
      if (kv_dtype == PA_F16 && q_dtype == PA_F16)
        return nt == 2 ? run(f16{}, f16{}, One{}, Yes{}, Yes{}) : run(f16{}, f16{}, Two{}, Yes{}, Yes{});
    }
    return PA_ERR_UNSUPPORTED;
  }
  if (kv_dtype == PA_BF16)
    return qf32 ? run(bf16{}, float{}, One{}, No{}, No{}) : run(bf16{}, bf16{}, One{}, No{}, No{});
  if (kv_dtype == PA_F16)
    return qf32 ? run(f16{}, float{}, One{}, No{}, No{}) : run(f16{}, f16{}, One{}, No{}, No{});
  if constexpr (D == 128) {  // an FP8 row of head_dim 128 fills one 128-byte TMA box
    if (q_dtype == PA_F32) return run(pa::fp8e4m3{}, float{}, One{}, No{}, No{});
    if (q_dtype == PA_F16) return run(pa::fp8e4m3{}, f16{}, One{}, No{}, No{});
    return run(pa::fp8e4m3{}, bf16{}, One{}, No{}, No{});
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int pa_set_option(int option, int value) {
  if (option == PA_OPT_WIDE_KERNEL && (value == PA_WIDE_MMA || value == PA_WIDE_TCGEN05 || value == PA_WIDE_AUTO)) {
    g_wide_kernel.store(value, std::memory_order_relaxed);
    return PA_OK;
  }
  if (option == PA_OPT_ITEM_SPLIT && (value == PA_SPLIT_ADAPTIVE || value == PA_SPLIT_FIXED)) {
    g_item_split.store(value, std::memory_order_relaxed);
    return PA_OK;
  }
  return PA_ERR_INVALID;
}

int pa_version(void) { return 101; }

const char* pa_strerror(int status) {
  switch (status) {
    case PA_OK: return "success";
    case PA_ERR_INVALID: return "invalid argument (null or misaligned pointer, or a size out of range)";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration (head_dim, block_size, dtype or group size)";
    case PA_ERR_WORKSPACE: return "workspace missing or smaller than pa_decode_workspace_size()";
    case PA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case PA_ERR_TOO_LARGE: return "the call needs more scratch than the built-in 64 MiB decode buffer";
    default: return "unknown pa_status";
  }
}

size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_seq_len,
                                int partition_size) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0 || partition_size < 0) return 0;
  const int P = partition_size ? partition_size : kDefaultPartition;
  return ws_layout(num_seqs, num_q_heads, head_dim, max_parts_for(max_seq_len, P)).total;
}

}  // extern "C"

namespace {

// pa_decode, pa_decode_fp8, pa_decode_multi and pa_decode_prefix: kv_dtype F16 / BF16 (scales
// unused) or FP8_E4M3; qtok query tokens per sequence (1 = decode); num_groups prefix groups
// (device int32 [num_groups][3]) whose shared items cover up to max_members sequences
int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                const int32_t* seq_lens, int num_seqs, int qtok, int num_q_heads, int num_kv_heads, int head_dim,
                int block_size, float scale, float k_scale, float v_scale, int max_blocks_per_seq,
                int64_t num_blocks, int q_dtype, int kv_dtype, int out_dtype, int partition_size,
                const int32_t* groups, int num_groups, int max_members, void* workspace, size_t workspace_bytes,
                void* stream) {
  if (num_seqs < 0 || qtok <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0 || partition_size < 0 || !std::isfinite(scale) ||
      !std::isfinite(k_scale) || !std::isfinite(v_scale) || k_scale <= 0.f || v_scale <= 0.f || num_groups < 0 ||
      max_members < 1)
    return PA_ERR_INVALID;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID;
  const int G = num_q_heads / num_kv_heads;
  if (G > 8 || num_kv_heads > 255) return PA_ERR_UNSUPPORTED;
  if (num_groups == 0) max_members = 1;
  if (max_members > 1 && qtok > 1) return PA_ERR_UNSUPPORTED;  // shared items are single-token decode
  // several query tokens: a 16-bit cache with a query of the same type
  if (qtok > 1 && (kv_dtype == PA_FP8_E4M3 || q_dtype != kv_dtype)) return PA_ERR_UNSUPPORTED;
  if (qtok > 65536 || static_cast<int64_t>(qtok) * num_q_heads * head_dim > INT_MAX) return PA_ERR_UNSUPPORTED;
  // items of more than 8 query rows may run on the tensor-core kernel (block size 16, head_dim 128,
  // a 16-bit cache with a query of its own type), which holds up to 64 rows per item: when it is
  // chosen, or by default when the rows per KV head exceed what the warp-MMA kernel's items hold
  // (that kernel would split the query tokens into column groups and read every page once per group)
  const int wide = g_wide_kernel.load(std::memory_order_relaxed);
  const bool tc_shape = head_dim == 128 && block_size == 16 && (kv_dtype == PA_F16 || kv_dtype == PA_BF16) &&
                        q_dtype == kv_dtype;
  const int64_t rows_wanted = static_cast<int64_t>(qtok) * max_members * G;
  const bool tc_ok = tc_shape && (wide == PA_WIDE_TCGEN05 ||
                                  (wide == PA_WIDE_AUTO && rows_wanted > max_item_rows(head_dim)));
  const int max_rows = tc_ok ? kTcMaxRows : max_item_rows(head_dim);
  // query tokens per item: all of them, or column groups of up to max_rows query rows per KV head
  // (8 with head_dim 64, whose items run on the one-consumer kernels)
  const int qtok_item = qtok * G <= max_rows ? qtok : std::max(1, max_rows / G);
  // an item holds qtok_item * G (or max_members * G) query rows: up to 8 on every dtype pair, up to
  // 32 (64 on the tensor-core kernel) on a 16-bit cache with a query of its own type and head_dim 128
  const int64_t cols = static_cast<int64_t>(qtok_item) * max_members * G;
  if (cols > max_rows) return PA_ERR_UNSUPPORTED;
  const bool use_tc = tc_ok && cols > 8;
  if (cols > 8 && (head_dim != 128 || kv_dtype == PA_FP8_E4M3 || q_dtype != kv_dtype)) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (kv_dtype == PA_FP8_E4M3) {
    if (head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (q_dtype != PA_F32 && q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  } else {
    if (kv_dtype != PA_F16 && kv_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (q_dtype != kv_dtype && q_dtype != PA_F32) return PA_ERR_UNSUPPORTED;
  }
  if (out_dtype != PA_F32 && out_dtype != PA_F16 && out_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  const int P = partition_size ? partition_size : kDefaultPartition;
  if (P % block_size || P / block_size > 32) return PA_ERR_UNSUPPORTED;
  if (num_blocks > INT_MAX / block_size) return PA_ERR_INVALID;
  const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  if (max_len > INT_MAX) return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || (num_groups && !groups))
    return PA_ERR_INVALID;
  if (num_groups > num_seqs) return PA_ERR_INVALID;  // disjoint groups of at least one sequence
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID;
  const int64_t max_parts = max_parts_for(max_len, P, num_groups > 0);
  if (max_parts > 32767) return PA_ERR_UNSUPPORTED;
  // partial results are kept per (query token, query head): the workspace of qtok * num_q_heads heads
  const WsLayout L = ws_layout(num_seqs, static_cast<int64_t>(qtok) * num_q_heads, head_dim, max_parts);
  if (!workspace || workspace_bytes < L.total) return PA_ERR_WORKSPACE;
  // the plan writes up to num_seqs * max_parts * ncg items (shared items of prefix groups take
  // partitions of their leader): they must fit the region the layout reserved for them
  const int64_t ncg = (qtok + qtok_item - 1) / qtok_item;
  if (static_cast<int64_t>(num_seqs) * max_parts * ncg * static_cast<int64_t>(sizeof(pa::WorkItem)) >
      static_cast<int64_t>(L.part_ml - L.items))
    return PA_ERR_WORKSPACE;
  const int64_t max_items = static_cast<int64_t>(num_seqs) * max_parts * ncg * num_kv_heads;
  if (max_items > INT_MAX) return PA_ERR_UNSUPPORTED;  // the kernels count (item, KV head) pairs in 32 bits
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PA_ERR_INVALID;

  int dev;
  DeviceInfo* info;
  if (current_device_info(&dev, &info) != PA_OK) return PA_ERR_CUDA;
  // a KV head row of two 128-byte column blocks (16-bit, head_dim 128) is fetched one page per box;
  // the tensor-core kernel reads K per column block (its S products take a chunk's rows of one block)
  const bool two = elem_bytes(kv_dtype) * head_dim == 256;
  CUtensorMap tmk, tmv, tmk_blocks;
  if (encode_kv_map(&tmk, k_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, two) != PA_OK ||
      encode_kv_map(&tmv, v_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, two) != PA_OK)
    return PA_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pa::DecodeParams p{};
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = G;
  p.head_dim = head_dim;
  p.block_size = block_size;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = static_cast<int>(num_blocks);
  p.partition_size = P;
  p.max_parts = static_cast<int>(max_parts);
  p.out_dtype = out_dtype;
  p.qtok = qtok;
  p.qtok_item = qtok_item;
  p.qbox_rows = qtok > 1 ? qtok_item : max_members;
  p.groups = groups;
  p.num_groups = num_groups;
  p.max_members = max_members;
  // items of up to four partitions, and the 128 pages a producer takes per item, where the plan
  // finds enough of them; one CTA per SM, with 4 rings (8 with an FP8 cache) or, on the
  // tensor-core kernel, one chunk pipeline
  const bool fp8 = kv_dtype == PA_FP8_E4M3;
  const bool fixed = g_item_split.load(std::memory_order_relaxed) == PA_SPLIT_FIXED;
  p.long_partition = fixed ? P : std::min(4 * P, 128 * block_size);
  p.rings = info->sm_count * (use_tc ? 1 : fp8 ? 8 : 4);
  p.scale_log2 = scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  p.v_scale = fp8 ? v_scale : 1.f;
  p.counters = reinterpret_cast<unsigned int*>(ws + L.counters);
  p.items = reinterpret_cast<pa::WorkItem*>(ws + L.items);
  p.seq_parts = reinterpret_cast<int*>(ws + L.seq_parts);
  p.seq_shared = reinterpret_cast<int*>(ws + L.seq_shared);
  p.seq_sub = reinterpret_cast<int*>(ws + L.seq_sub);
  p.part_ml = reinterpret_cast<float2*>(ws + L.part_ml);
  p.part_acc = reinterpret_cast<float*>(ws + L.part_acc);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pa::pa_decode_plan_kernel<<<1, pa::kPlanThreads, 0, st>>>(p);
  if (cudaPeekAtLastError() != cudaSuccess) return PA_ERR_CUDA;

  int rc;
  const int c = static_cast<int>(cols);
  CUtensorMap tmq;
  if (use_tc && (encode_q_map(&tmq, q, q_dtype, static_cast<int64_t>(num_seqs) * qtok, num_q_heads, G,
                              p.qbox_rows) != PA_OK ||
                 encode_k_tc_map(&tmk_blocks, k_cache, kv_dtype, num_blocks, block_size, num_kv_heads) != PA_OK))
    return PA_ERR_CUDA;
  const CUtensorMap* tq = use_tc ? &tmq : nullptr;
  if (block_size == 16)
    rc = head_dim == 128
             ? dispatch_kv<16, 128>(p, tmk, tmv, tq, &tmk_blocks, max_items, dev, info, kv_dtype, q_dtype, c, st)
             : dispatch_kv<16, 64>(p, tmk, tmv, tq, &tmk_blocks, max_items, dev, info, kv_dtype, q_dtype, c, st);
  else
    rc = head_dim == 128
             ? dispatch_kv<32, 128>(p, tmk, tmv, tq, &tmk_blocks, max_items, dev, info, kv_dtype, q_dtype, c, st)
             : dispatch_kv<32, 64>(p, tmk, tmv, tq, &tmk_blocks, max_items, dev, info, kv_dtype, q_dtype, c, st);
  if (rc != PA_OK) return rc;
  {  // merge kernel: waits (griddepcontrol.wait) for the partition kernel's partial results
    const int64_t warps = static_cast<int64_t>(num_seqs) * qtok * num_q_heads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((warps + pa::kMergeWarps - 1) / pa::kMergeWarps));
    cfg.blockDim = dim3(pa::kMergeWarps * 32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, pa::pa_decode_merge_kernel, p) != cudaSuccess) return PA_ERR_CUDA;
  }
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

extern "C" {

int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
              const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, float scale, int max_blocks_per_seq, int64_t num_blocks, int q_dtype,
              int kv_dtype, int out_dtype, int partition_size, void* workspace, size_t workspace_bytes,
              void* stream) {
  if (kv_dtype == PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;  // needs its scales: pa_decode_fp8
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, 1, num_q_heads, num_kv_heads,
                     head_dim, block_size, scale, 1.f, 1.f, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype,
                     out_dtype, partition_size, nullptr, 0, 1, workspace, workspace_bytes, stream);
}

int pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                  const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                  int block_size, float scale, float k_scale, float v_scale, int max_blocks_per_seq,
                  int64_t num_blocks, int q_dtype, int out_dtype, int partition_size, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, 1, num_q_heads, num_kv_heads,
                     head_dim, block_size, scale, k_scale, v_scale, max_blocks_per_seq, num_blocks, q_dtype,
                     PA_FP8_E4M3, out_dtype, partition_size, nullptr, 0, 1, workspace, workspace_bytes, stream);
}

int pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    const int32_t* seq_lens, int num_seqs, int num_q_tokens, int num_q_heads, int num_kv_heads,
                    int head_dim, int block_size, float scale, int max_blocks_per_seq, int64_t num_blocks,
                    int q_dtype, int kv_dtype, int out_dtype, int partition_size, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (kv_dtype == PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_q_tokens, num_q_heads,
                     num_kv_heads, head_dim, block_size, scale, 1.f, 1.f, max_blocks_per_seq, num_blocks, q_dtype,
                     kv_dtype, out_dtype, partition_size, nullptr, 0, 1, workspace, workspace_bytes, stream);
}

int pa_decode_prefix(void* out, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                     int64_t num_blocks, int q_dtype, int kv_dtype, int out_dtype, int partition_size,
                     const int32_t* prefix_groups, int num_groups, int max_members, void* workspace,
                     size_t workspace_bytes, void* stream) {
  if (kv_dtype == PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, 1, num_q_heads, num_kv_heads,
                     head_dim, block_size, scale, 1.f, 1.f, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype,
                     out_dtype, partition_size, prefix_groups, num_groups, max_members, workspace,
                     workspace_bytes, stream);
}

int pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                         int kv_dtype, int64_t k_token_stride, int64_t v_token_stride, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
      k_token_stride < 0 || v_token_stride < 0)
    return PA_ERR_INVALID;
  if (kv_dtype != PA_F16 && kv_dtype != PA_BF16 && kv_dtype != PA_F32) return PA_ERR_UNSUPPORTED;
  const int es = elem_bytes(kv_dtype);
  const int64_t row = static_cast<int64_t>(num_kv_heads) * head_dim;
  if ((row * es) % 16) return PA_ERR_UNSUPPORTED;
  if (!k_token_stride) k_token_stride = row;
  if (!v_token_stride) v_token_stride = row;
  if (k_token_stride < row || v_token_stride < row || (k_token_stride * es) % 16 || (v_token_stride * es) % 16)
    return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID;
  int dev;
  DeviceInfo* info;
  if (current_device_info(&dev, &info) != PA_OK) return PA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(num_tokens, 64LL * info->sm_count));
  pa::pa_reshape_and_cache_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(k), static_cast<const uint8_t*>(v), static_cast<uint8_t*>(k_cache),
      static_cast<uint8_t*>(v_cache), slot_mapping, num_tokens, row * es, k_token_stride * es, v_token_stride * es,
      num_blocks * block_size);
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int64_t num_blocks, int in_dtype, float k_scale, float v_scale,
                             int64_t k_token_stride, int64_t v_token_stride, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
      k_token_stride < 0 || v_token_stride < 0 || !std::isfinite(k_scale) || !std::isfinite(v_scale) ||
      k_scale <= 0.f || v_scale <= 0.f)
    return PA_ERR_INVALID;
  if (in_dtype != PA_F32 && in_dtype != PA_F16 && in_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (row % 16) return PA_ERR_UNSUPPORTED;  // 8 elements per thread, 16-byte aligned cache rows
  if (!k_token_stride) k_token_stride = row;
  if (!v_token_stride) v_token_stride = row;
  if (k_token_stride < row || v_token_stride < row) return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  const int es = elem_bytes(in_dtype);
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v) || (k_token_stride * es) % 16 ||
      (v_token_stride * es) % 16)
    return PA_ERR_INVALID;
  int dev;
  DeviceInfo* info;
  if (current_device_info(&dev, &info) != PA_OK) return PA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(num_tokens, 64LL * info->sm_count));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* kc = static_cast<uint8_t*>(k_cache);
  uint8_t* vc = static_cast<uint8_t*>(v_cache);
  const int64_t slots = num_blocks * block_size;
  if (in_dtype == PA_BF16)
    pa::pa_reshape_and_cache_fp8_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), kc, vc, slot_mapping, num_tokens,
        row, k_token_stride, v_token_stride, slots, k_scale, v_scale);
  else if (in_dtype == PA_F16)
    pa::pa_reshape_and_cache_fp8_kernel<__half><<<grid, 128, 0, st>>>(
        static_cast<const __half*>(k), static_cast<const __half*>(v), kc, vc, slot_mapping, num_tokens, row,
        k_token_stride, v_token_stride, slots, k_scale, v_scale);
  else
    pa::pa_reshape_and_cache_fp8_kernel<float><<<grid, 128, 0, st>>>(
        static_cast<const float*>(k), static_cast<const float*>(v), kc, vc, slot_mapping, num_tokens, row,
        k_token_stride, v_token_stride, slots, k_scale, v_scale);
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst_pairs, int num_pairs, int64_t num_blocks,
                   size_t block_bytes, const int32_t* host_pairs, void* stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0 || block_bytes % 16) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !src_dst_pairs) return PA_ERR_INVALID;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID;
  if (host_pairs) {
    std::unordered_set<int32_t> dsts, srcs;
    for (int i = 0; i < num_pairs; ++i) {
      const int32_t s = host_pairs[2 * i], d = host_pairs[2 * i + 1];
      if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks || s == d) return PA_ERR_INVALID;
      if (!dsts.insert(d).second) return PA_ERR_INVALID;
      srcs.insert(s);
    }
    for (int32_t d : dsts)
      if (srcs.count(d)) return PA_ERR_INVALID;
  }
  const int64_t vecs = static_cast<int64_t>(block_bytes / 16);
  // chunks of 4 vectors per thread (a 32 KB block: 2 chunks of 256 threads)
  const int chunks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(16, vecs / (256 * 4))));
  pa::pa_copy_blocks_kernel<<<dim3(static_cast<unsigned>(num_pairs), 2, static_cast<unsigned>(chunks)), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(static_cast<uint8_t*>(k_cache),
                                                                   static_cast<uint8_t*>(v_cache), src_dst_pairs,
                                                                   num_blocks, static_cast<int64_t>(block_bytes));
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache, const void* src_v_cache,
                   const int32_t* src_dst_pairs, int num_pairs, int64_t num_src_blocks, int64_t num_dst_blocks,
                   size_t block_bytes, void* stream) {
  if (num_pairs < 0 || num_src_blocks <= 0 || num_dst_blocks <= 0 || block_bytes == 0 || block_bytes % 16)
    return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !src_dst_pairs) return PA_ERR_INVALID;
  if (!aligned16(dst_k_cache) || !aligned16(dst_v_cache) || !aligned16(src_k_cache) || !aligned16(src_v_cache))
    return PA_ERR_INVALID;
  const int64_t vecs = static_cast<int64_t>(block_bytes / 16);
  const int chunks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(16, vecs / (256 * 4))));
  pa::pa_swap_blocks_kernel<<<dim3(static_cast<unsigned>(num_pairs), 2, static_cast<unsigned>(chunks)), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint8_t*>(dst_k_cache), static_cast<uint8_t*>(dst_v_cache), static_cast<const uint8_t*>(src_k_cache),
      static_cast<const uint8_t*>(src_v_cache), src_dst_pairs, num_src_blocks, num_dst_blocks,
      static_cast<int64_t>(block_bytes));
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_selftest_wait_timeout(int polls, void* stream) {
  if (polls < 1 || polls > static_cast<int>(pa::kWaitLimit)) return PA_ERR_INVALID;
  pa::pa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t>(polls));
  return cudaPeekAtLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int code = 0;
  if (cudaMemcpyFromSymbol(&code, pa::g_dev_error, sizeof(code)) != cudaSuccess) return PA_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(pa::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  return static_cast<int>(code);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// pa_decode_static_workspace: pa_decode with its scratch in a device global of this file, for
// callers that cannot allocate device memory when they decode (see include/pa.h).
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_pa_static_workspace[PA_DECODE_STATIC_WORKSPACE_BYTES];

namespace {
void* g_static_ws_addr[kMaxDevices];  // device address of g_pa_static_workspace, per device
std::mutex g_static_ws_mu;
}  // namespace

extern "C" int pa_decode_static_workspace(void* out, const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                          int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                          float scale, int max_blocks_per_seq, int64_t num_blocks, int q_dtype,
                                          int kv_dtype, int out_dtype, int partition_size, void* stream) {
  // argument errors are reported by pa_decode itself; only the size limit is checked here
  if (num_seqs > 0 && num_q_heads > 0 && head_dim > 0 && block_size > 0 && max_blocks_per_seq > 0 &&
      partition_size >= 0) {
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * block_size;
    if (max_len <= INT_MAX) {
      const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, static_cast<int>(max_len),
                                                   partition_size);
      if (need > PA_DECODE_STATIC_WORKSPACE_BYTES) return PA_ERR_TOO_LARGE;
    }
  }
  void* ws = nullptr;
  if (num_seqs > 0) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_static_ws_mu);
    if (!g_static_ws_addr[dev]) {  // once per device, with that device current
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_pa_static_workspace) != cudaSuccess || !addr) return PA_ERR_CUDA;
      g_static_ws_addr[dev] = addr;
    }
    ws = g_static_ws_addr[dev];
  }
  return pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                   block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, out_dtype, partition_size,
                   ws, ws ? PA_DECODE_STATIC_WORKSPACE_BYTES : 0, stream);
}
