// libpagedkv: the C ABI declared in include/pagedkv.h.
//
// Host side only: argument validation (before any CUDA call), resolution of the
// split-context partition size, workspace layout, and kernel launches.  The
// kernels live in decode.cuh (paged decode attention: plan, persistent decode
// with the log-sum-exp merge of split contexts) and cache_ops.cuh (append, block
// copy, gather).
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_set>
#include <vector>

#include <cudaTypedefs.h>

#include "pagedkv.h"
#include "pkv_device.cuh"
#include "decode.cuh"
#include "decode_gqa.cuh"
#include "multi_query_tc.cuh"
#include "gqa_tc.cuh"
#include "cache_ops.cuh"

namespace {

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int elem_bytes(pkv_dtype dt) {
  switch (dt) {
    case PKV_F32: return 4;
    case PKV_F16: return 2;
    case PKV_BF16: return 2;
  }
  return 0;
}

bool head_dim_ok(int d) { return d == 64 || d == 128; }
bool block_size_ok(int b) { return b == 8 || b == 16 || b == 32 || b == 64 || b == 128; }

size_t round16(size_t x) { return (x + 15) / 16 * 16; }

// ---------------------------------------------------------------------------
// Decode plan: partition size and workspace layout.
// ---------------------------------------------------------------------------
struct DecodePlan {
  int part_tokens = 0;
  int max_parts = 1;
  bool split = false;
  bool sort = false;
  size_t off_units = 0, off_ml = 0, off_acc = 0, bytes = 0;
};

// Library choice of partition size when the caller passes 0.  The persistent
// grid holds about kRefCtas CTAs (148 SMs x 2).  When there are at least 4 (sequence,
// head) units per CTA and no context exceeds 4096 tokens, the longest-first unit
// order already balances the CTAs and splitting would only add partial-state
// traffic and a merge launch, so contexts are not split (measured on B200: the
// batch-256 OPT-13B layer and the batch-64 LLaMA-7B layer both run 4-6% faster
// unsplit).  Otherwise contexts are cut into 512-token partitions (a multiple of
// every supported block size), which bounds the work of one unit.  Maximum
// contexts of at most 512 tokens are never split.
constexpr int kAutoPartitionTokens = 512;
constexpr long long kRefCtas = 148 * 2;
// The plan kernel orders the units longest first for up to kPlanThreads sequences
// (one thread per sequence, any number of partitions) and for unit lists up to
// this length (one warp, 32 sequences per step; the lengths are staged in shared
// memory).
constexpr long long kSortedUnitsMax = pkv::kPlanSortMaxSeqs;

// H = partial-state rows per sequence (query heads x query tokens); Hkv = work
// units per (sequence, partition) counted by the no-split decision (K/V heads, so
// that the decision does not depend on which kernel runs).
int make_plan(int S, int H, int Hkv, int D, int B, int MB, int requested, DecodePlan* plan) {
  if (S < 0 || H <= 0 || MB <= 0) return PKV_EINVAL;
  if (Hkv <= 0) return PKV_EINVAL;
  if (!head_dim_ok(D) || !block_size_ok(B)) return PKV_EUNSUPPORTED;
  if (S > 65535 || H > 65535) return PKV_EINVAL;
  const long long max_ctx = (long long)MB * B;
  if (max_ctx > (INT_MAX / 2)) return PKV_EINVAL;
  if (requested < 0 || (requested > 0 && requested % B != 0)) return PKV_EINVAL;
  long long pt = requested;
  if (requested == 0) {
    const bool enough_units = (long long)S * Hkv >= 4 * kRefCtas && max_ctx <= 4096;
    pt = (max_ctx <= kAutoPartitionTokens || enough_units) ? max_ctx : kAutoPartitionTokens;
  }
  if (pt >= max_ctx) pt = max_ctx;
  const long long parts = (max_ctx + pt - 1) / pt;
  if (parts > 32767) return PKV_EINVAL;
  if ((long long)S * H * parts > (long long)INT_MAX / 2) return PKV_EINVAL;
  plan->part_tokens = (int)pt;
  plan->max_parts = (int)parts;
  plan->split = parts > 1;
  plan->sort = S <= pkv::kPlanThreads || (long long)S * parts <= kSortedUnitsMax;
  size_t off = 16;  // counters[2] (+ padding)
  plan->off_units = off;
  off += round16((size_t)S * parts * sizeof(uint2));
  if (plan->split) {
    plan->off_ml = off;
    off += round16((size_t)S * H * parts * sizeof(float2));
    plan->off_acc = off;
    off += round16((size_t)S * H * parts * D * sizeof(float));
  }
  plan->bytes = off;
  return PKV_OK;
}

// ---------------------------------------------------------------------------
// Per-device launch facts, filled on first use.
// ---------------------------------------------------------------------------
std::mutex g_mu;
int g_sm_count[kMaxDevices];

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return PKV_ECUDA;
  return PKV_OK;
}

int sm_count(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// Resident CTAs per SM of one decode instantiation (after raising its shared-memory limit).
template <typename T, int D, int TT, int NS>
int decode_occupancy(int dev) {
  static int occ[kMaxDevices];
  std::lock_guard<std::mutex> lk(g_mu);
  if (occ[dev] == 0) {
    using Tr = pkv::DecodeTraits<T, D, TT, NS>;
    auto kern = pkv::paged_decode_kernel<T, D, TT, NS>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::kSmemBytes) != cudaSuccess)
      return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kDecodeThreads, Tr::kSmemBytes) !=
            cudaSuccess ||
        n <= 0)
      return 0;
    occ[dev] = n;
  }
  return occ[dev];
}

template <typename T, int D, int TT, int NS>
int launch_decode(const pkv::DecodeParams& prm, long long max_units, cudaStream_t st) {
  using Tr = pkv::DecodeTraits<T, D, TT, NS>;
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  const int sms = sm_count(dev);
  const int occ = decode_occupancy<T, D, TT, NS>(dev);
  if (sms <= 0 || occ <= 0) return PKV_ECUDA;
  long long grid = (long long)sms * occ;
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  // Programmatic dependent launch: the CTAs start while the plan kernel runs and
  // wait for it (griddepcontrol.wait) after their prologue.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(pkv::kDecodeThreads);
  cfg.dynamicSmemBytes = Tr::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_decode_kernel<T, D, TT, NS>, prm) != cudaSuccess) return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// Tile sizes: every stage holds 32 KB of K+V (64 rows of 256 bytes for 16-bit
// D=128).  16-bit K/V with at least kShallowRingUnits (sequence, head,
// partition) units runs two stages per CTA and three CTAs per SM; fewer units
// run three stages and two CTAs per SM.  The shallow ring keeps the same bytes in
// flight per SM but gives it three independent unit streams, so the SM crosses
// unit boundaries (a block-table and list-entry round trip each) more often in
// parallel, and more sequences that share prefix blocks run at the same time and
// meet in L2.  With few units the longest one becomes the critical path, and a
// CTA's share of HBM bandwidth shrinks with every extra CTA.  Measured on B200
// (bf16/fp16, D=128, B=16): three CTAs per SM are 1-4% faster for batch 64-256
// OPT-13B layers, 17% at B=8, 22% for the shared-prefix sampling batch and 6%
// for a batch-128 LLaMA-7B layer; 8-10% slower at 1280 and 2048 units.
constexpr long long kShallowRingUnits = 8 * kRefCtas;

template <int D>
int dispatch_decode(pkv_dtype dt, const pkv::DecodeParams& prm, long long max_units, cudaStream_t st) {
  constexpr int kTT16 = 16384 / (D * 2);
  constexpr int kTT32 = 16384 / (D * 4);
  const bool shallow = max_units >= kShallowRingUnits;
  switch (dt) {
    case PKV_F16:
      return shallow ? launch_decode<__half, D, kTT16, 2>(prm, max_units, st)
                     : launch_decode<__half, D, kTT16, 3>(prm, max_units, st);
    case PKV_BF16:
      return shallow ? launch_decode<__nv_bfloat16, D, kTT16, 2>(prm, max_units, st)
                     : launch_decode<__nv_bfloat16, D, kTT16, 3>(prm, max_units, st);
    case PKV_F32: return launch_decode<float, D, kTT32, 3>(prm, max_units, st);
  }
  return PKV_EDTYPE;
}

// ---------------------------------------------------------------------------
// Grouped-query tensor-core kernel: tensor maps over the pools and the launch.
// ---------------------------------------------------------------------------
std::mutex g_tmap_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  if (g_encode_tiled == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return PKV_ECUDA;
    g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode_tiled;
  return PKV_OK;
}

// 2-D view of one pool: rows = num_blocks * Hkv * B, columns = D (16-bit); boxes of
// 64 columns x box_rows rows, 128-byte swizzle.
int encode_pool_map(CUtensorMap* map, const void* pool, long long rows, int D, int box_rows, pkv_dtype dt) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (tensor_map_encoder(&enc) != PKV_OK) return PKV_ECUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t elem_strides[2] = {1, 1};
  const CUtensorMapDataType type =
      dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = enc(map, type, 2, const_cast<void*>(pool), dims, strides, box, elem_strides,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ECUDA;
}

template <typename T, int D, int NS>
int launch_gqa(const pkv::GqaParams& prm, long long max_units, cudaStream_t st) {
  using Tr = pkv::GqaTraits<D, NS>;
  static int occ[kMaxDevices];
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  const int sms = sm_count(dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (occ[dev] == 0) {
      auto kern = pkv::paged_decode_gqa_kernel<T, D, NS>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::kSmemAlloc) != cudaSuccess)
        return PKV_ECUDA;
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, pkv::kDecodeThreads, Tr::kSmemAlloc) !=
              cudaSuccess ||
          n <= 0)
        return PKV_ECUDA;
      occ[dev] = n;
    }
  }
  if (sms <= 0) return PKV_ECUDA;
  long long grid = (long long)sms * occ[dev];
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(pkv::kDecodeThreads);
  cfg.dynamicSmemBytes = Tr::kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_decode_gqa_kernel<T, D, NS>, prm) != cudaSuccess) return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// Whether the tensor-core grouped-query kernel serves these arguments.
bool use_gqa_kernel(int Hq, int Hkv, int B, int NB, pkv_dtype dt) {
  const int G = Hq / Hkv;
  return G >= 2 && G <= pkv::kGqaRows && dt != PKV_F32 && (long long)NB * Hkv * B < (1LL << 31);
}

// Which tensor-core kernel serves Lq * G query rows per K/V head (16-bit K/V):
//  * kKt: the token-major tcgen05 kernel (gqa_tc.cuh), head_dim 128 and
//    kKtMinRows < Lq * G <= kKtMaxRows: all rows of a (sequence, K/V head) in one
//    row tile, the tile's tokens as M;
//  * kTc128: the row-major tcgen05 kernel (multi_query_tc.cuh) above that (or
//    head_dim 64 above 16 rows): 128-row tiles of floor(128 / G) whole query tokens;
//  * kMmaSync: the warp-level kernel (decode_gqa.cuh), 16-row tiles.
// Measured on B200 (batch-256 layer, 8 K/V heads x 128, bf16, attention call): the
// token-major kernel is ahead from 8 rows (G = 8: 5.56 vs 5.49 TB/s; G = 16: 5.52
// vs 4.94; 16 rows of a 4-token verify: 5.47 vs 4.94) and behind below (G = 2:
// 5.48 vs 5.87; G = 4: 5.48 vs 5.79).
// The choice depends only on the shapes, so the workspace query and the launch agree.
enum class TcPath { kMmaSync, kKt, kTc128 };
constexpr long long kKtMinRows = 7;
constexpr long long kKtMaxRows = 64;

TcPath tc_path(long long q_len, int group, int head_dim) {
  const long long rows = q_len * group;
  if (head_dim == 128 && rows > kKtMinRows && rows <= kKtMaxRows) return TcPath::kKt;
  if (rows > pkv::kGqaRows && group <= pkv::kTcRows && (head_dim == 64 || head_dim == 128)) return TcPath::kTc128;
  return TcPath::kMmaSync;
}

bool mq_uses_tcgen05(long long q_len, int group, int head_dim) {
  return tc_path(q_len, group, head_dim) != TcPath::kMmaSync;
}

long long mq_row_tiles(long long q_len, int group, int head_dim) {
  const TcPath path = tc_path(q_len, group, head_dim);
  if (path == TcPath::kKt) return 1;
  if (path == TcPath::kTc128) {
    const long long tq = pkv::kTcRows / group;
    return (q_len + tq - 1) / tq;
  }
  return (q_len * group + pkv::kGqaRows - 1) / pkv::kGqaRows;
}

// Launch the tensor-core kernel for Lq query tokens per sequence over the plan's
// unit list (the plan kernel has been launched already).
int launch_tensor_core(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                       const int32_t* context_lens, int num_seqs, int q_len, int num_heads, int num_kv_heads,
                       int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype,
                       float scale_log2, float* out, const DecodePlan& plan, const pkv::DecodeParams& prm,
                       cudaStream_t st) {
  static_assert(alignof(pkv::GqaParams) >= 64, "tensor maps need 64-byte alignment");
  pkv::GqaParams g;
  const long long rows = (long long)num_blocks * num_kv_heads * block_size;
  const int box_rows = block_size < pkv::kGqaTile ? block_size : pkv::kGqaTile;
  if (encode_pool_map(&g.tmap_k, k_cache, rows, head_dim, box_rows, dtype) != PKV_OK ||
      encode_pool_map(&g.tmap_v, v_cache, rows, head_dim, box_rows, dtype) != PKV_OK)
    return PKV_ECUDA;
  g.q = q;
  g.block_tables = block_tables;
  g.context_lens = context_lens;
  g.num_heads = num_heads;
  g.num_kv_heads = num_kv_heads;
  g.group = num_heads / num_kv_heads;
  g.q_len = q_len;
  g.rows = q_len * g.group;
  g.row_tiles = (g.rows + pkv::kGqaRows - 1) / pkv::kGqaRows;
  g.block_size = block_size;
  g.max_blocks = max_blocks_per_seq;
  g.num_blocks = num_blocks;
  g.scale_log2 = scale_log2;
  g.part_tokens = plan.part_tokens;
  g.max_parts = plan.max_parts;
  g.out = out;
  g.ws_acc = prm.ws_acc;
  g.ws_ml = prm.ws_ml;
  g.units = prm.units;
  g.counters = prm.counters;
  const long long max_units = (long long)num_seqs * num_kv_heads * g.row_tiles * plan.max_parts;
  if (dtype == PKV_BF16)
    return head_dim == 64 ? launch_gqa<__nv_bfloat16, 64, 3>(g, max_units, st)
                          : launch_gqa<__nv_bfloat16, 128, 3>(g, max_units, st);
  return head_dim == 64 ? launch_gqa<__half, 64, 3>(g, max_units, st) : launch_gqa<__half, 128, 3>(g, max_units, st);
}

// 4-D view [S][Lq][Hq][D] of the query rows (16-bit); boxes of 64 columns x G heads
// x Tq tokens x 1 sequence, 128-byte swizzle, so that one box lands as the
// 128-byte-swizzled rows r = token * G + head of a 128-row operand tile.
int encode_query_map(CUtensorMap* map, const void* q, int S, int Lq, int Hq, int D, int G, int Tq, pkv_dtype dt) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  if (tensor_map_encoder(&enc) != PKV_OK) return PKV_ECUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)Lq, (cuuint64_t)S};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2, (cuuint64_t)Lq * Hq * D * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)Tq, 1};
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  const CUtensorMapDataType type =
      dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = enc(map, type, 4, const_cast<void*>(q), dims, strides, box, elem_strides,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ECUDA;
}

template <typename T, int D>
int launch_tc(const pkv::TcParams& prm, long long max_units, cudaStream_t st) {
  using Tr = pkv::TcTraits<D>;
  static bool attr_set[kMaxDevices];
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  const int sms = sm_count(dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(pkv::paged_multi_query_tc_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Tr::kSmemAlloc) != cudaSuccess)
        return PKV_ECUDA;
      attr_set[dev] = true;
    }
  }
  if (sms <= 0) return PKV_ECUDA;
  long long grid = (long long)sms * pkv::kTcCtasPerSm;  // resident CTAs (shared memory and tensor memory)
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(pkv::kTcThreads);
  cfg.dynamicSmemBytes = Tr::kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_multi_query_tc_kernel<T, D>, prm) != cudaSuccess) return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int launch_tcgen05(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables, int num_seqs,
                   int q_len, int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                   int num_blocks, pkv_dtype dtype, float scale_log2, float* out, const DecodePlan& plan,
                   const pkv::DecodeParams& prm, cudaStream_t st) {
  static_assert(alignof(pkv::TcParams) >= 64, "tensor maps need 64-byte alignment");
  pkv::TcParams t;
  const int G = num_heads / num_kv_heads;
  const int Tq = pkv::kTcRows / G;
  const long long rows = (long long)num_blocks * num_kv_heads * block_size;
  const int box_rows = block_size < pkv::kTcTile ? block_size : pkv::kTcTile;
  if (encode_pool_map(&t.tmap_k, k_cache, rows, head_dim, box_rows, dtype) != PKV_OK ||
      encode_pool_map(&t.tmap_v, v_cache, rows, head_dim, box_rows, dtype) != PKV_OK ||
      encode_query_map(&t.tmap_q, q, num_seqs, q_len, num_heads, head_dim, G, Tq, dtype) != PKV_OK)
    return PKV_ECUDA;
  t.block_tables = block_tables;
  t.num_heads = num_heads;
  t.num_kv_heads = num_kv_heads;
  t.group = G;
  t.q_len = q_len;
  t.tq_per_tile = Tq;
  t.row_tiles = (int)mq_row_tiles(q_len, G, head_dim);
  t.block_size = block_size;
  t.max_blocks = max_blocks_per_seq;
  t.num_blocks = num_blocks;
  t.scale_log2 = scale_log2;
  t.part_tokens = plan.part_tokens;
  t.max_parts = plan.max_parts;
  t.out = out;
  t.ws_acc = prm.ws_acc;
  t.ws_ml = prm.ws_ml;
  t.units = prm.units;
  t.counters = prm.counters;
  const long long max_units = (long long)num_seqs * num_kv_heads * t.row_tiles * plan.max_parts;
  if (dtype == PKV_BF16)
    return head_dim == 64 ? launch_tc<__nv_bfloat16, 64>(t, max_units, st) : launch_tc<__nv_bfloat16, 128>(t, max_units, st);
  return head_dim == 64 ? launch_tc<__half, 64>(t, max_units, st) : launch_tc<__half, 128>(t, max_units, st);
}

template <typename T, int NR>
int launch_kt(const pkv::TcParams& prm, long long max_units, cudaStream_t st) {
  using Tr = pkv::KtTraits<NR>;
  static bool attr_set[kMaxDevices];
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  const int sms = sm_count(dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(pkv::paged_gqa_tc_kernel<T, NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Tr::kSmemAlloc) != cudaSuccess)
        return PKV_ECUDA;
      attr_set[dev] = true;
    }
  }
  if (sms <= 0) return PKV_ECUDA;
  long long grid = sms;  // one CTA per SM (shared memory)
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(pkv::kKtThreads);
  cfg.dynamicSmemBytes = Tr::kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_gqa_tc_kernel<T, NR>, prm) != cudaSuccess) return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// The token-major tcgen05 kernel: all Lq * G <= 64 rows of a (sequence, K/V head)
// in one row tile of NR = 16, 32 or 64 rows; 128-token K/V tiles.
int launch_kt_path(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables, int num_seqs,
                   int q_len, int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                   int num_blocks, pkv_dtype dtype, float scale_log2, float* out, const DecodePlan& plan,
                   const pkv::DecodeParams& prm, cudaStream_t st) {
  static_assert(alignof(pkv::TcParams) >= 64, "tensor maps need 64-byte alignment");
  pkv::TcParams t;
  const int G = num_heads / num_kv_heads;
  const int rows = q_len * G;
  const long long pool_rows = (long long)num_blocks * num_kv_heads * block_size;
  const int box_rows = block_size < pkv::kKtTile ? block_size : pkv::kKtTile;
  if (encode_pool_map(&t.tmap_k, k_cache, pool_rows, head_dim, box_rows, dtype) != PKV_OK ||
      encode_pool_map(&t.tmap_v, v_cache, pool_rows, head_dim, box_rows, dtype) != PKV_OK ||
      encode_query_map(&t.tmap_q, q, num_seqs, q_len, num_heads, head_dim, G, q_len, dtype) != PKV_OK)
    return PKV_ECUDA;
  t.block_tables = block_tables;
  t.num_heads = num_heads;
  t.num_kv_heads = num_kv_heads;
  t.group = G;
  t.q_len = q_len;
  t.tq_per_tile = q_len;
  t.row_tiles = 1;
  t.block_size = block_size;
  t.max_blocks = max_blocks_per_seq;
  t.num_blocks = num_blocks;
  t.scale_log2 = scale_log2;
  t.part_tokens = plan.part_tokens;
  t.max_parts = plan.max_parts;
  t.out = out;
  t.ws_acc = prm.ws_acc;
  t.ws_ml = prm.ws_ml;
  t.units = prm.units;
  t.counters = prm.counters;
  const long long max_units = (long long)num_seqs * num_kv_heads * plan.max_parts;
  const bool bf = dtype == PKV_BF16;
  if (rows <= 16)
    return bf ? launch_kt<__nv_bfloat16, 16>(t, max_units, st) : launch_kt<__half, 16>(t, max_units, st);
  if (rows <= 32)
    return bf ? launch_kt<__nv_bfloat16, 32>(t, max_units, st) : launch_kt<__half, 32>(t, max_units, st);
  return bf ? launch_kt<__nv_bfloat16, 64>(t, max_units, st) : launch_kt<__half, 64>(t, max_units, st);
}

// The plan kernel is a programmatic dependent of the stream's previous kernel: it
// reads the context lengths and sorts while that kernel finishes, and waits for it
// before writing the unit list and the counters.
int launch_plan(const int32_t* context_lens, int num_seqs, int max_ctx, const DecodePlan& plan, uint2* units,
                int* counters, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(pkv::kPlanThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_decode_plan_kernel, context_lens, num_seqs, max_ctx, plan.part_tokens,
                         plan.sort ? 1 : 0, units, counters) != cudaSuccess)
    return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// The merge is a programmatic dependent of the decode kernel: its CTAs may be
// scheduled as decode CTAs run out of units and wait for the decode to finish.
template <int D>
int launch_merge(const int32_t* context_lens, int S, int H, int max_ctx, const DecodePlan& plan, const float* ws_acc,
                 const float2* ws_ml, float* out, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)H, (unsigned)S);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pkv::paged_decode_merge_kernel<D>, context_lens, H, max_ctx, plan.part_tokens,
                         plan.max_parts, ws_acc, ws_ml, out) != cudaSuccess)
    return PKV_ECUDA;
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// Debug checks of the cache-maintenance inputs: -1 until first queried, then 0 / 1.
std::atomic<int> g_debug_checks{-1};

bool debug_checks() {
  int v = g_debug_checks.load();
  if (v < 0) {
    const char* e = std::getenv("PKV_CHECK");
    int want = (e && e[0] == '1' && e[1] == 0) ? 1 : 0;
    g_debug_checks.compare_exchange_strong(v, want);
    v = g_debug_checks.load();
  }
  return v == 1;
}

// Copies device (or any CUDA-visible) memory to a host array, in stream order.
int copy_to_host(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return PKV_OK;
  if (cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, st) != cudaSuccess) return PKV_ECUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int grid_for(long long work, int per_block, int dev) {
  long long blocks = (work + per_block - 1) / per_block;
  const int sms = sm_count(dev);
  const long long cap = (long long)(sms > 0 ? sms : 148) * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

size_t paged_attn_decode_workspace_size(int num_seqs, int num_heads, int head_dim, int block_size,
                                        int max_blocks_per_seq, int partition_tokens) {
  DecodePlan plan;
  if (make_plan(num_seqs, num_heads, num_heads, head_dim, block_size, max_blocks_per_seq, partition_tokens,
                &plan) != PKV_OK)
    return (size_t)-1;
  return plan.bytes;
}

int paged_attn_decode_partition_tokens(int num_seqs, int num_heads, int head_dim, int block_size,
                                       int max_blocks_per_seq, int partition_tokens) {
  DecodePlan plan;
  const int rc = make_plan(num_seqs, num_heads, num_heads, head_dim, block_size, max_blocks_per_seq,
                           partition_tokens, &plan);
  return rc != PKV_OK ? rc : plan.part_tokens;
}

}  // extern "C"

namespace {

// Paged decode for num_heads query heads over num_kv_heads K/V heads (equal for
// multi-head attention).  Shared by every decode entry point.
int decode_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype, float scale, float* out,
                int partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  if (elem_bytes(dtype) == 0) return PKV_EDTYPE;
  if (num_kv_heads <= 0 || num_heads <= 0 || num_heads % num_kv_heads != 0) return PKV_EINVAL;
  DecodePlan plan;
  const int rc = make_plan(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           partition_tokens, &plan);
  if (rc != PKV_OK) return rc;
  if (num_blocks <= 0) return PKV_EINVAL;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_EINVAL;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_EALIGN;
  if (workspace && (!aligned(workspace, 16) || workspace_bytes < plan.bytes)) {
    return aligned(workspace, 16) ? PKV_EWORKSPACE : PKV_EALIGN;
  }

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool owned = false;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), plan.bytes, st) != cudaSuccess) return PKV_ECUDA;
    owned = true;
  }

  pkv::DecodeParams prm;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.num_heads = num_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.group = num_heads / num_kv_heads;
  prm.block_size = block_size;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_blocks = num_blocks;
  prm.scale_log2 = scale * pkv::kLog2e;
  prm.part_tokens = plan.part_tokens;
  prm.max_parts = plan.max_parts;
  prm.out = out;
  prm.ws_acc = plan.split ? reinterpret_cast<float*>(ws + plan.off_acc) : nullptr;
  prm.ws_ml = plan.split ? reinterpret_cast<float2*>(ws + plan.off_ml) : nullptr;
  prm.units = reinterpret_cast<const uint2*>(ws + plan.off_units);
  prm.counters = reinterpret_cast<int*>(ws);

  const int max_ctx = max_blocks_per_seq * block_size;
  int result = PKV_OK;
  if (launch_plan(context_lens, num_seqs, max_ctx, plan, reinterpret_cast<uint2*>(ws + plan.off_units), prm.counters,
                  st) != PKV_OK)
    result = PKV_ECUDA;
  const int group = num_heads / num_kv_heads;
  const bool tc_ok = dtype != PKV_F32 && group >= 2 && (long long)num_blocks * num_kv_heads * block_size < (1LL << 31);
  if (result == PKV_OK && tc_ok && tc_path(1, group, head_dim) == TcPath::kKt) {
    result = launch_kt_path(q, k_cache, v_cache, block_tables, num_seqs, 1, num_heads, num_kv_heads, head_dim,
                            block_size, max_blocks_per_seq, num_blocks, dtype, prm.scale_log2, out, plan, prm, st);
  } else if (result == PKV_OK && use_gqa_kernel(num_heads, num_kv_heads, block_size, num_blocks, dtype)) {
    result = launch_tensor_core(q, k_cache, v_cache, block_tables, context_lens, num_seqs, 1, num_heads,
                                num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, dtype, prm.scale_log2,
                                out, plan, prm, st);
  } else if (result == PKV_OK && dtype != PKV_F32 && mq_uses_tcgen05(1, num_heads / num_kv_heads, head_dim) &&
             (long long)num_blocks * num_kv_heads * block_size < (1LL << 31)) {
    // more than 16 query heads per K/V head: one 128-row tcgen05 tile per (sequence, K/V head)
    result = launch_tcgen05(q, k_cache, v_cache, block_tables, num_seqs, 1, num_heads, num_kv_heads, head_dim,
                            block_size, max_blocks_per_seq, num_blocks, dtype, prm.scale_log2, out, plan, prm, st);
  } else if (result == PKV_OK) {
    const long long max_units = (long long)num_seqs * num_heads * plan.max_parts;
    result = head_dim == 64 ? dispatch_decode<64>(dtype, prm, max_units, st)
                            : dispatch_decode<128>(dtype, prm, max_units, st);
  }
  if (result == PKV_OK && plan.split) {
    result = head_dim == 64
                 ? launch_merge<64>(context_lens, num_seqs, num_heads, max_ctx, plan, prm.ws_acc, prm.ws_ml, out, st)
                 : launch_merge<128>(context_lens, num_seqs, num_heads, max_ctx, plan, prm.ws_acc, prm.ws_ml, out, st);
  }
  if (owned && cudaFreeAsync(ws, st) != cudaSuccess && result == PKV_OK) result = PKV_ECUDA;
  return result;
}

// Several query tokens per sequence (tensor-core kernels only: 16-bit K/V).
int multi_query_plan(int num_seqs, int q_len, int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int partition_tokens, DecodePlan* plan) {
  if (q_len <= 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return PKV_EINVAL;
  const long long row_tiles = mq_row_tiles(q_len, num_heads / num_kv_heads, head_dim);
  if (row_tiles > 32767 || (long long)q_len * num_heads > 65535) return PKV_EINVAL;
  return make_plan(num_seqs, q_len * num_heads, (int)(num_kv_heads * row_tiles), head_dim, block_size,
                   max_blocks_per_seq, partition_tokens, plan);
}

int multi_query_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int num_seqs, int q_len, int num_heads, int num_kv_heads,
                     int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype,
                     float scale, float* out, int partition_tokens, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (elem_bytes(dtype) == 0) return PKV_EDTYPE;
  if (dtype == PKV_F32) return PKV_EUNSUPPORTED;
  DecodePlan plan;
  const int rc = multi_query_plan(num_seqs, q_len, num_heads, num_kv_heads, head_dim, block_size,
                                  max_blocks_per_seq, partition_tokens, &plan);
  if (rc != PKV_OK) return rc;
  if (num_blocks <= 0) return PKV_EINVAL;
  if ((long long)num_blocks * num_kv_heads * block_size >= (1LL << 31)) return PKV_EINVAL;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_EINVAL;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_EALIGN;
  if (workspace && (!aligned(workspace, 16) || workspace_bytes < plan.bytes)) {
    return aligned(workspace, 16) ? PKV_EWORKSPACE : PKV_EALIGN;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool owned = false;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), plan.bytes, st) != cudaSuccess) return PKV_ECUDA;
    owned = true;
  }
  pkv::DecodeParams prm = {};
  prm.ws_acc = plan.split ? reinterpret_cast<float*>(ws + plan.off_acc) : nullptr;
  prm.ws_ml = plan.split ? reinterpret_cast<float2*>(ws + plan.off_ml) : nullptr;
  prm.units = reinterpret_cast<const uint2*>(ws + plan.off_units);
  prm.counters = reinterpret_cast<int*>(ws);
  const int max_ctx = max_blocks_per_seq * block_size;
  int result = PKV_OK;
  if (launch_plan(context_lens, num_seqs, max_ctx, plan, reinterpret_cast<uint2*>(ws + plan.off_units), prm.counters,
                  st) != PKV_OK)
    result = PKV_ECUDA;
  const TcPath path = tc_path(q_len, num_heads / num_kv_heads, head_dim);
  if (result == PKV_OK && path == TcPath::kKt)
    result = launch_kt_path(q, k_cache, v_cache, block_tables, num_seqs, q_len, num_heads, num_kv_heads, head_dim,
                            block_size, max_blocks_per_seq, num_blocks, dtype, scale * pkv::kLog2e, out, plan, prm,
                            st);
  else if (result == PKV_OK && path == TcPath::kTc128)
    result = launch_tcgen05(q, k_cache, v_cache, block_tables, num_seqs, q_len, num_heads, num_kv_heads, head_dim,
                            block_size, max_blocks_per_seq, num_blocks, dtype, scale * pkv::kLog2e, out, plan, prm,
                            st);
  else if (result == PKV_OK)
    result = launch_tensor_core(q, k_cache, v_cache, block_tables, context_lens, num_seqs, q_len, num_heads,
                                num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, dtype,
                                scale * pkv::kLog2e, out, plan, prm, st);
  if (result == PKV_OK && plan.split) {
    // partial states are kept per (sequence, query token, query head): q_len * num_heads rows per sequence
    result = head_dim == 64 ? launch_merge<64>(context_lens, num_seqs, q_len * num_heads, max_ctx, plan, prm.ws_acc,
                                               prm.ws_ml, out, st)
                            : launch_merge<128>(context_lens, num_seqs, q_len * num_heads, max_ctx, plan,
                                                prm.ws_acc, prm.ws_ml, out, st);
  }
  if (owned && cudaFreeAsync(ws, st) != cudaSuccess && result == PKV_OK) result = PKV_ECUDA;
  return result;
}

}  // namespace

extern "C" {

int paged_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_seqs, int num_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int num_blocks, pkv_dtype dtype, float scale, float* out,
                      int partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_heads, head_dim,
                     block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, partition_tokens, workspace,
                     workspace_bytes, stream);
}

size_t paged_attn_decode_gqa_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                            int block_size, int max_blocks_per_seq, int partition_tokens) {
  DecodePlan plan;
  if (make_plan(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, partition_tokens,
                &plan) != PKV_OK)
    return (size_t)-1;
  return plan.bytes;
}

size_t paged_attn_multi_query_workspace_size(int num_seqs, int q_len, int num_heads, int num_kv_heads,
                                             int head_dim, int block_size, int max_blocks_per_seq,
                                             int partition_tokens) {
  DecodePlan plan;
  if (multi_query_plan(num_seqs, q_len, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       partition_tokens, &plan) != PKV_OK)
    return (size_t)-1;
  return plan.bytes;
}

int paged_attn_multi_query(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs, int q_len, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype,
                           float scale, float* out, int partition_tokens, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return multi_query_impl(q, k_cache, v_cache, block_tables, context_lens, num_seqs, q_len, num_heads, num_kv_heads,
                          head_dim, block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, partition_tokens,
                          workspace, workspace_bytes, stream);
}

int paged_attn_decode_tune(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype, float scale,
                           float* out, void* workspace, size_t workspace_bytes, int reps, float* times_ms,
                           int* candidates, int max_candidates, int* num_candidates, void* stream) {
  if (reps <= 0 || reps > 1000 || !workspace || max_candidates < 0) return PKV_EINVAL;
  // candidates: no split, then 4096 ... 64 tokens that split the maximum context
  const long long max_ctx = (long long)max_blocks_per_seq * block_size;
  if (max_ctx <= 0 || max_ctx > INT_MAX / 2) return PKV_EINVAL;
  int cand[8];
  int nc = 0;
  cand[nc++] = (int)max_ctx;
  for (int pt = 4096; pt >= 64; pt /= 2)
    if (pt % block_size == 0 && pt < max_ctx && nc < 8) cand[nc++] = pt;
  for (int i = 0; i < nc; ++i) {
    const size_t need = paged_attn_decode_gqa_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                             max_blocks_per_seq, cand[i]);
    if (need == (size_t)-1) return PKV_EINVAL;
    if (need > workspace_bytes) return PKV_EWORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return PKV_ECUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return PKV_ECUDA;
  }
  int best = -1;
  float best_ms = 0.f;
  int rc = PKV_OK;
  for (int i = 0; i < nc && rc == PKV_OK; ++i) {
    // one untimed call, then `reps` timed back-to-back calls
    for (int r = 0; r <= reps && rc == PKV_OK; ++r) {
      if (r == 1 && cudaEventRecord(e0, st) != cudaSuccess) rc = PKV_ECUDA;
      if (rc == PKV_OK)
        rc = decode_impl(q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
                         head_dim, block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, cand[i], workspace,
                         workspace_bytes, stream);
    }
    float ms = 0.f;
    if (rc == PKV_OK && (cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
                         cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess))
      rc = PKV_ECUDA;
    if (rc != PKV_OK) break;
    ms /= reps;
    if (times_ms && i < max_candidates) times_ms[i] = ms;
    if (candidates && i < max_candidates) candidates[i] = cand[i];
    if (best < 0 || ms < best_ms) {
      best = cand[i];
      best_ms = ms;
    }
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (num_candidates) *num_candidates = nc;
  if (rc != PKV_OK) return rc;
  // leave `out` holding the result of the chosen partition size
  rc = decode_impl(q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                   block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, best, workspace, workspace_bytes,
                   stream);
  return rc != PKV_OK ? rc : best;
}

size_t paged_attn_decode_tune_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                             int block_size, int max_blocks_per_seq) {
  // the smallest candidate partition needs the largest workspace
  const long long max_ctx = (long long)max_blocks_per_seq * block_size;
  if (max_ctx <= 0 || max_ctx > INT_MAX / 2) return (size_t)-1;
  size_t most = paged_attn_decode_gqa_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                     max_blocks_per_seq, 0);
  if (most == (size_t)-1) return most;
  for (int pt = 4096; pt >= 64; pt /= 2) {
    if (pt % block_size || pt >= max_ctx) continue;
    const size_t n = paged_attn_decode_gqa_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                          max_blocks_per_seq, pt);
    if (n == (size_t)-1) return n;
    if (n > most) most = n;
  }
  return most;
}

int paged_attn_decode_gqa_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq, int partition_tokens) {
  DecodePlan plan;
  const int rc = make_plan(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           partition_tokens, &plan);
  return rc != PKV_OK ? rc : plan.part_tokens;
}

int paged_attn_decode_gqa(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                          int block_size, int max_blocks_per_seq, int num_blocks, pkv_dtype dtype, float scale,
                          float* out, int partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                     block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, partition_tokens, workspace,
                     workspace_bytes, stream);
}

int pkv_check_copy_pairs(const int64_t* host_pairs, int num_pairs) {
  if (num_pairs < 0 || (num_pairs > 0 && !host_pairs)) return PKV_EINVAL;
  std::unordered_set<int64_t> srcs, dsts;
  for (int i = 0; i < num_pairs; ++i) {
    if (host_pairs[2 * i] < 0 || host_pairs[2 * i + 1] < 0) continue;  // skipped by the copy kernel
    srcs.insert(host_pairs[2 * i]);
    if (host_pairs[2 * i] == host_pairs[2 * i + 1] || !dsts.insert(host_pairs[2 * i + 1]).second)
      return PKV_EOVERLAP;
  }
  for (int64_t d : dsts)
    if (srcs.count(d)) return PKV_EOVERLAP;
  return PKV_OK;
}

int pkv_check_slots(const int64_t* host_slots, int num_tokens) {
  if (num_tokens < 0 || (num_tokens > 0 && !host_slots)) return PKV_EINVAL;
  std::unordered_set<int64_t> seen;
  for (int i = 0; i < num_tokens; ++i)
    if (host_slots[i] >= 0 && !seen.insert(host_slots[i]).second) return PKV_EOVERLAP;
  return PKV_OK;
}

int pkv_set_debug_checks(int enable) {
  const int before = debug_checks() ? 1 : 0;
  if (enable >= 0) g_debug_checks.store(enable ? 1 : 0);
  return before;
}

int kv_cache_append(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                    int num_tokens, int num_heads, int head_dim, int block_size, int num_blocks, pkv_dtype dtype,
                    void* stream) {
  const int e = elem_bytes(dtype);
  if (e == 0) return PKV_EDTYPE;
  if (num_tokens < 0 || num_heads <= 0 || num_blocks <= 0) return PKV_EINVAL;
  if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PKV_EUNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_EINVAL;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PKV_EALIGN;
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  (void)dev;
  const int row_vecs = head_dim * e / 16;
  if ((long long)num_heads * row_vecs > INT_MAX) return PKV_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (debug_checks()) {
    std::vector<int64_t> h((size_t)num_tokens);
    const int rc = copy_to_host(h.data(), slot_mapping, h.size() * sizeof(int64_t), st);
    if (rc != PKV_OK) return rc;
    const int ck = pkv_check_slots(h.data(), num_tokens);
    if (ck != PKV_OK) return ck;
  }
  pkv::kv_append_kernel<<<dim3((unsigned)num_tokens, 2), pkv::kAppendThreads, 0, st>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_heads, row_vecs, block_size,
      (long long)num_blocks * block_size);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int kv_block_copy(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs, int num_heads,
                  int head_dim, int block_size, int num_blocks, pkv_dtype dtype, void* stream) {
  const int e = elem_bytes(dtype);
  if (e == 0) return PKV_EDTYPE;
  if (num_pairs < 0 || num_heads <= 0 || num_blocks <= 0) return PKV_EINVAL;
  if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PKV_EUNSUPPORTED;
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !src_dst_pairs) return PKV_EINVAL;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(src_dst_pairs, 8)) return PKV_EALIGN;
  const long long block_vecs = (long long)num_heads * block_size * head_dim * e / 16;
  const long long per_cta = (long long)pkv::kCopyThreads * pkv::kCopyVecs;
  const long long chunks = (block_vecs + per_cta - 1) / per_cta;
  if (chunks > INT_MAX) return PKV_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (debug_checks()) {
    std::vector<int64_t> h(2 * (size_t)num_pairs);
    const int rc = copy_to_host(h.data(), src_dst_pairs, h.size() * sizeof(int64_t), st);
    if (rc != PKV_OK) return rc;
    const int ck = pkv_check_copy_pairs(h.data(), num_pairs);
    if (ck != PKV_OK) return ck;
  }
  for (int first = 0; first < num_pairs; first += 65535) {
    const int n = num_pairs - first < 65535 ? num_pairs - first : 65535;
    const dim3 grid((unsigned)chunks, (unsigned)n, 2);
    pkv::kv_block_copy_kernel<<<grid, pkv::kCopyThreads, 0, st>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), src_dst_pairs + 2 * (size_t)first, block_vecs,
        num_blocks);
    if (cudaGetLastError() != cudaSuccess) return PKV_ECUDA;
  }
  return PKV_OK;
}

}  // extern "C"

namespace {

// Device address of pinned host memory, or nullptr if `p` is not page-locked host memory.
void* pinned_device_address(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  return a.devicePointer;
}

int swap_impl(void* k_cache, void* v_cache, void* host_k, void* host_v, const int64_t* block_ids, int n,
              int num_heads, int head_dim, int block_size, int num_blocks, pkv_dtype dtype, void* stream,
              int to_host) {
  const int e = elem_bytes(dtype);
  if (e == 0) return PKV_EDTYPE;
  if (n < 0 || num_heads <= 0 || num_blocks <= 0) return PKV_EINVAL;
  if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PKV_EUNSUPPORTED;
  if (n == 0) return PKV_OK;
  if (!k_cache || !v_cache || !host_k || !host_v || !block_ids) return PKV_EINVAL;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(host_k, 16) || !aligned(host_v, 16) ||
      !aligned(block_ids, 8))
    return PKV_EALIGN;
  if (n > 65535) return PKV_EINVAL;
  void* dk = pinned_device_address(host_k);
  void* dv = pinned_device_address(host_v);
  if (!dk || !dv) return PKV_EINVAL;
  const long long block_vecs = (long long)num_heads * block_size * head_dim * e / 16;
  const long long per_cta = (long long)pkv::kCopyThreads * pkv::kCopyVecs;
  const long long chunks = (block_vecs + per_cta - 1) / per_cta;
  if (chunks > INT_MAX) return PKV_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  pkv::kv_swap_kernel<<<dim3((unsigned)chunks, (unsigned)n, 2), pkv::kCopyThreads, 0, st>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<uint4*>(dk), static_cast<uint4*>(dv),
      block_ids, block_vecs, num_blocks, to_host);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

}  // namespace

extern "C" {

int kv_blocks_to_host(const void* k_cache, const void* v_cache, const int64_t* block_ids, int num_blocks_moved,
                      void* host_k, void* host_v, int num_heads, int head_dim, int block_size, int num_blocks,
                      pkv_dtype dtype, void* stream) {
  return swap_impl(const_cast<void*>(k_cache), const_cast<void*>(v_cache), host_k, host_v, block_ids,
                   num_blocks_moved, num_heads, head_dim, block_size, num_blocks, dtype, stream, 1);
}

int kv_blocks_from_host(const void* host_k, const void* host_v, void* k_cache, void* v_cache, const int64_t* block_ids,
                        int num_blocks_moved, int num_heads, int head_dim, int block_size, int num_blocks,
                        pkv_dtype dtype, void* stream) {
  return swap_impl(k_cache, v_cache, const_cast<void*>(host_k), const_cast<void*>(host_v), block_ids,
                   num_blocks_moved, num_heads, head_dim, block_size, num_blocks, dtype, stream, 0);
}

int paged_kv_gather(const void* cache, const int32_t* block_table_row, int context_len, int num_heads, int head_dim,
                    int block_size, int num_blocks, pkv_dtype dtype, void* out, void* stream) {
  const int e = elem_bytes(dtype);
  if (e == 0) return PKV_EDTYPE;
  if (context_len < 0 || num_heads <= 0 || num_blocks <= 0) return PKV_EINVAL;
  if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PKV_EUNSUPPORTED;
  if (context_len == 0) return PKV_OK;
  if (!cache || !block_table_row || !out) return PKV_EINVAL;
  if (!aligned(cache, 16) || !aligned(out, 16) || !aligned(block_table_row, 4)) return PKV_EALIGN;
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  const int row_vecs = head_dim * e / 16;
  const long long total = (long long)num_heads * context_len * row_vecs;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  pkv::kv_gather_kernel<<<grid_for(total, 256, dev), 256, 0, st>>>(
      static_cast<const uint4*>(cache), block_table_row, context_len, num_heads, row_vecs, block_size, num_blocks,
      static_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_get_device_error(void* stream, int* reason) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (reason) *reason = PKV_DEV_OK;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKV_ECUDA;
  int word = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&word, pkv::g_error_word, sizeof(int), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return PKV_ECUDA;
  if (cudaMemcpyToSymbolAsync(pkv::g_error_word, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return PKV_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKV_ECUDA;
  if (reason) *reason = word;
  if (word == PKV_DEV_OK) return PKV_OK;
  return word == PKV_DEV_WAIT_TIMEOUT ? PKV_ETIMEOUT : PKV_EDEVICE;
}

int pkv_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > pkv::kWaitLimitCycles) return PKV_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int minus_one = -1;
  if (cudaMemcpyToSymbolAsync(pkv::g_selftest_waited_out, &minus_one, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return PKV_ECUDA;
  pkv::wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(limit_cycles);
  if (cudaGetLastError() != cudaSuccess) return PKV_ECUDA;
  int waited_out = -1;
  if (cudaMemcpyFromSymbolAsync(&waited_out, pkv::g_selftest_waited_out, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return PKV_ECUDA;
  return waited_out == 1 ? 1 : (waited_out == 0 ? 0 : PKV_ECUDA);
}

const char* pkv_strerror(int code) {
  switch (code) {
    case PKV_OK: return "success";
    case PKV_EINVAL: return "invalid argument (null pointer, size out of range or bad partition size)";
    case PKV_EDTYPE: return "unknown storage dtype";
    case PKV_EALIGN: return "pointer not aligned as required (16 bytes for data, 4/8 for indices)";
    case PKV_EUNSUPPORTED: return "head_dim or block_size not supported";
    case PKV_ECUDA: return "CUDA runtime call or kernel launch failed";
    case PKV_EWORKSPACE: return "workspace smaller than paged_attn_decode_workspace_size()";
    case PKV_EDEVICE: return "a kernel flagged bad device data (block id, context length, slot or copy pair)";
    case PKV_ETIMEOUT: return "a kernel's bounded shared-memory wait ran out";
    case PKV_ENOMEM: return "block manager: not enough free blocks (nothing was changed)";
    case PKV_ESEQ: return "block manager: unknown sequence, sequence already exists, or repeated in a batch";
    case PKV_EOVERLAP: return "debug checks: copy pairs overlap, or two appended tokens share a slot";
  }
  return "unknown error code";
}

int pkv_abi_version(void) { return 1; }

}  // extern "C"

// ---------------------------------------------------------------------------
// paged_attn_decode_noalloc: the decode with its scratch in a static device
// array, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------
namespace {

// The scratch every paged_attn_decode_noalloc call on a device shares.  In host
// code this name is only a stand-in for the device array; its device address
// comes from cudaGetSymbolAddress (below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (the first call on a device does it) and cached.
int noalloc_scratch(void** ptr) {
  int dev;
  if (current_device(&dev) != PKV_OK) return PKV_ECUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return PKV_ECUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return PKV_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                                         int num_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                         int num_blocks, pkv_dtype dtype, float scale, float* out,
                                         int partition_tokens, void* stream) {
  // The argument checks of paged_attn_decode, in its order, so that both entry
  // points return the same code for the same arguments; the scratch array then
  // plays the part of a caller workspace of PKV_NOALLOC_SCRATCH_BYTES.
  if (elem_bytes(dtype) == 0) return PKV_EDTYPE;
  if (num_heads <= 0) return PKV_EINVAL;
  DecodePlan plan;
  const int prc = make_plan(num_seqs, num_heads, num_heads, head_dim, block_size, max_blocks_per_seq,
                            partition_tokens, &plan);
  if (prc != PKV_OK) return prc;
  if (num_blocks <= 0) return PKV_EINVAL;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_EINVAL;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_EALIGN;
  if (plan.bytes > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_EWORKSPACE;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != PKV_OK) return rc;
  return paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, head_dim,
                           block_size, max_blocks_per_seq, num_blocks, dtype, scale, out, partition_tokens, scratch,
                           (size_t)PKV_NOALLOC_SCRATCH_BYTES, stream);
}
