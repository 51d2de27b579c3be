// Paged single-query decode attention for sm_100a.
//
// Three kernels, launched back to back on one stream:
//
//  1. paged_decode_plan_kernel (one CTA): turns context_lens into a compact list
//     of live (sequence, partition) work units, each with its sequence's clamped
//     context length, longest first when the list is short enough to sort in one
//     CTA, and resets the unit counter.
//  2. paged_decode_kernel (persistent, launched as a programmatic dependent of
//     the plan so that its prologue overlaps it): CTA b starts with unit b, then
//     takes units from the counter until none are left.  A unit is (sequence s,
//     head h, partition p).
//     The CTA streams the unit's K and V rows through a ring of NS shared-memory
//     stages:
//       producer warp  follows the block table and issues one bulk (TMA-engine)
//                      copy per contiguous (block, head) run of rows, plus the q
//                      row at a unit's first tile; it writes a small header per
//                      stage (unit, valid rows, first/last flags) and announces
//                      the stage's bytes on its "full" mbarrier.  It reads the
//                      table before waiting for a free stage and fetches the next
//                      unit's list entry (which carries the context length) while
//                      streaming the current one, so the ring does not drain
//                      between units.
//       4 consumer warps   each 8-lane group takes one token at a time: a lane
//                      owns D/8 dimensions, reads its 16-byte chunks of the K row
//                      from shared memory, and the group reduces q.k with three
//                      xor-shuffles.  Each group keeps its own online-softmax
//                      state (running max m, running sum l, unnormalised
//                      accumulator) in base 2, rescaled once per tile, and adds
//                      its tokens' V rows.  At a unit's last tile the groups and
//                      warps merge their states exactly and write either the
//                      final row (single-partition context) or the partition's
//                      (m, l, acc) to the workspace.
//  3. paged_decode_merge_kernel (programmatic dependent of the decode kernel):
//     log-sum-exp merge of the partitions of every (sequence, head) whose context
//     spans more than one partition,
//       M = max_p m_p,  L = sum_p l_p 2^(m_p - M),  out = sum_p acc_p 2^(m_p - M) / L,
//     which is exact algebra.
//
// The method follows each sequence's block table to its scattered physical blocks
// and attends over them as if they were one contiguous context
// ("PagedAttention - Efficient Memory Management for LLM Serving with vLLM",
// section "Method (PagedAttention + vLLM)").  Here the gather is done by the
// copy engine straight into shared memory, so each K/V byte crosses HBM once.
// One query per sequence makes this ~1 flop per byte: HBM-bound, no tensor cores.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kTileFirst = 1, kTileLast = 2, kTileEnd = 4 };

template <typename T, int D, int TT, int NS>
struct DecodeTraits {
  static constexpr int kE = sizeof(T);
  static constexpr int kRowBytes = D * kE;
  static constexpr int kPerChunk = Elem<T>::kPerChunk;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kChunksPerLane = kChunksPerRow / 8;  // 8 lanes share one row
  static constexpr int kDimsPerLane = kChunksPerLane * kPerChunk;
  static constexpr int kGroups = kConsumerWarps * 4;  // 8-lane groups per CTA
  static constexpr int kTokPerGroup = TT / kGroups;   // tokens per group per tile
  static constexpr int kTileBytes = TT * kRowBytes;   // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQOffset = NS * kStageBytes;              // NS q rows
  static constexpr int kHdrOffset = kQOffset + NS * kRowBytes;   // NS int4 headers
  static constexpr int kBarOffset = kHdrOffset + NS * 16;        // full[NS], empty[NS], epi
  static constexpr int kAbortOffset = kBarOffset + (2 * NS + 1) * 8;
  static constexpr int kRedOffset = (kAbortOffset + 16 + 15) / 16 * 16;
  static constexpr int kRedFloats = kConsumerWarps * (D + 2);    // one buffer
  static constexpr int kSmemBytes = kRedOffset + 2 * kRedFloats * 4;
  static_assert(kRowBytes % 128 == 0, "a row must split into 8 lanes x 16-byte chunks");
  static_assert(TT % kGroups == 0, "every group gets the same number of tokens per tile");
  static_assert((TT & (TT - 1)) == 0 && TT >= 16, "tile tokens: a power of two >= 16");
  static_assert(TT / 8 <= 32, "at most one copy unit per producer lane");
  static_assert(D <= kConsumerWarps * 32, "the final merge gives each consumer thread <= 1 dimension");
};

// (d0, d1) += (a0, a1) * (b0, b1): two fp32 fused multiply-adds in one packed
// instruction (sm_100); each lane rounds exactly as fmaf does, so results are the
// same as two fmaf calls with half the instructions.
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t d, a, b;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

// d0 += a.lo * b.lo and d1 += a.hi * b.hi for two packed 16-bit pairs, accumulated in
// fp32 (mixed-precision FMA, sm_100): the product of two 16-bit values is exact in fp32 and
// each sum is rounded once, as fmaf on the widened values would be, with no widening step.
template <typename T>
struct MixedFma;
template <>
struct MixedFma<__nv_bfloat16> {
  static __device__ __forceinline__ void pair(uint32_t a, uint32_t b, float& d0, float& d1) {
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %2;\n\t"
        "mov.b32 {b0, b1}, %3;\n\t"
        "fma.rn.f32.bf16 %0, a0, b0, %0;\n\t"
        "fma.rn.f32.bf16 %1, a1, b1, %1;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "r"(a), "r"(b));
  }
};
template <>
struct MixedFma<__half> {
  static __device__ __forceinline__ void pair(uint32_t a, uint32_t b, float& d0, float& d1) {
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %2;\n\t"
        "mov.b32 {b0, b1}, %3;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
        "fma.rn.f32.f16 %1, a1, b1, %1;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "r"(a), "r"(b));
  }
};

struct DecodeParams {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int num_heads;      // query heads (Hq)
  int num_kv_heads;   // K/V heads in the pools (Hkv); query head h reads K/V head h / group
  int group;          // Hq / Hkv
  int block_size;
  int max_blocks;
  int num_blocks;
  float scale_log2;   // scale * log2(e): logits are kept in base 2
  int part_tokens;    // tokens per partition; >= max_blocks * block_size when not splitting
  int max_parts;      // partitions a context can span (workspace stride)
  float* out;         // [S][H][D]
  float* ws_acc;      // [S][H][max_parts][D]   (split only)
  float2* ws_ml;      // [S][H][max_parts]      (split only)
  const uint2* units;     // {(s << 16) | p, clamped context length} per live (sequence, partition)
  int* counters;          // [0] unit counter, [1] number of live (sequence, partition)
};

__device__ __forceinline__ int clamp_ctx(int ctx, int max_ctx) { return ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx); }

// Number of partitions a context of ctx tokens occupies; an empty context still
// gets one unit so that its output row is written (as zeros).
__device__ __forceinline__ int parts_of(int ctx, int part_tokens) {
  const int n = (ctx + part_tokens - 1) / part_tokens;
  return n < 1 ? 1 : n;
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// 1. plan (one CTA).  With `sort`, the units are ordered by decreasing length
//    (unit_bucket) with a stable counting sort: within a bucket the units keep
//    (sequence, partition) order, so sequences that share prefix blocks stay
//    adjacent and their shared blocks are re-read from L2.  Longest-first lets
//    the dynamically scheduled CTAs end together.  Up to kPlanThreads sequences
//    are placed in one pass, one thread per sequence; longer lists take one warp
//    over runs of 32 sequences.  The plan is a programmatic dependent launch: it
//    reads the lengths and sorts while the stream's previous kernel finishes (our
//    kernels let dependents start early; none writes the lengths), and waits for
//    that kernel before its first write, so it never changes the list or the
//    counters under a previous call's decode kernel.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 128;
constexpr int kPlanSortMaxSeqs = 4096;  // sorted lists: num_seqs * partitions <= this
static_assert(kPlanBuckets % 32 == 0, "the bucket scan gives every lane the same number of buckets");
static_assert(kPlanThreads == 1024 && kPlanBuckets == 128, "one-pass sort: 32 warps, eight threads per key");

// Sort key of a unit of len tokens, non-decreasing in len: 8-token buckets up to
// 512 tokens, 256-token buckets above (the last bucket takes everything past
// 16.4K).  The units claimed last decide how evenly the CTAs end and they are
// the shortest, so the short end is sorted finely (a unit of 250 tokens holds a
// CTA ~6 us); above it the wide buckets keep sequences of similar length in
// submission order, so that samples sharing prefix blocks run side by side.
__device__ __forceinline__ int unit_bucket(int len) {
  if (len <= 512) return (len + 7) >> 3;                                  // 0 .. 64
  return min(kPlanBuckets - 1, 64 + ((len - 512 + 255) >> 8));            // 65 .. 127
}

// One pass of the stable counting sort with one thread per sequence (num_seqs <=
// kPlanThreads).  A sequence's partitions but the last are full (bucket
// key_full); its last partition has bucket key.  Bucket key_full holds its units
// in (sequence, partition) order: unit (s, p) sits after every unit of the
// sequences before s in that bucket (an exclusive scan over the sequences).
// Any other bucket holds last partitions only, in sequence order: the rank of s
// among the sequences with its key is its rank within its warp (match_any)
// plus the count of that key in the warps before (a scan over the 32 warps).
__device__ __forceinline__ void plan_sort_one_pass(const int32_t* __restrict__ context_lens, int num_seqs,
                                                   int max_ctx, int part_tokens, uint2* __restrict__ units,
                                                   int* __restrict__ counters) {
  constexpr int kWarps = kPlanThreads / 32;
  __shared__ int cnt[kWarps][kPlanBuckets];  // per warp and key: count, then exclusive offset
  __shared__ int total[kPlanBuckets];        // sequences whose last partition has key k
  __shared__ int start[kPlanBuckets];        // first position of bucket k
  __shared__ int wsum[kWarps];               // per warp: units in bucket key_full, then exclusive prefix
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int s = tid;
  const bool live = s < num_seqs;
  int ctx = 0;
  if (live) {
    const int raw = context_lens[s];
    if (raw < 0 || raw > max_ctx) flag_error(PKV_DEV_CONTEXT_LEN);
    ctx = clamp_ctx(raw, max_ctx);
  }
  const int n = live ? parts_of(ctx, part_tokens) : 0;
  const int nfull = max(n - 1, 0);
  const int key_full = unit_bucket(part_tokens);
  const int key = live ? unit_bucket(ctx - (n - 1) * part_tokens) : -1;
  for (int i = tid; i < kWarps * kPlanBuckets; i += kPlanThreads) (&cnt[0][0])[i] = 0;
  // this sequence's units in bucket key_full, scanned over the warp
  const int gv = nfull + (key == key_full ? 1 : 0);
  int g_incl = gv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, g_incl, o);
    if (lane >= o) g_incl += v;
  }
  const unsigned same = __match_any_sync(0xffffffffu, key);
  const int rank = __popc(same & ((1u << lane) - 1u));
  __syncthreads();  // cnt is zero
  if (live && rank == 0) cnt[warp][key] = __popc(same);
  if (lane == 31) wsum[warp] = g_incl;
  __syncthreads();
  {
    // key k = tid / 8: eight threads scan its counts over the warps, four warps each
    const int k = tid >> 3, q = tid & 7;
    int c[kWarps / 8];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kWarps / 8; ++i) {
      c[i] = cnt[(kWarps / 8) * q + i][k];
      sum += c[i];
    }
    int sc = sum;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, sc, o, 8);
      if (q >= o) sc += v;
    }
    int ex = sc - sum;
#pragma unroll
    for (int i = 0; i < kWarps / 8; ++i) {
      cnt[(kWarps / 8) * q + i][k] = ex;
      ex += c[i];
    }
    if (q == 7) total[k] = sc;
  }
  int g_total = 0;
  if (warp == 0) {
    // exclusive prefix of the warps' key_full units
    const int w = wsum[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    g_total = __shfl_sync(0xffffffffu, wi, 31);
    __syncwarp();
    wsum[lane] = wi - w;
  }
  __syncthreads();
  // the previous call's kernels may still read the list and the counters
  pdl_wait_primary();
  if (warp == 0) {
    // bucket starts, longest bucket first: lane l owns buckets 127-4l ... 124-4l
    int c[kPlanBuckets / 32];
    int mine = 0;
#pragma unroll
    for (int j = 0; j < kPlanBuckets / 32; ++j) {
      const int k = kPlanBuckets - 1 - (kPlanBuckets / 32) * lane - j;
      c[j] = k == key_full ? g_total : total[k];
      mine += c[j];
    }
    int excl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, excl, o);
      if (lane >= o) excl += v;
    }
    const int all = __shfl_sync(0xffffffffu, excl, 31);
    excl -= mine;
#pragma unroll
    for (int j = 0; j < kPlanBuckets / 32; ++j) {
      start[kPlanBuckets - 1 - (kPlanBuckets / 32) * lane - j] = excl;
      excl += c[j];
    }
    if (lane == 0) {
      counters[0] = 0;
      counters[1] = all;
    }
  }
  __syncthreads();
  if (live) {
    const int at_full = start[key_full] + wsum[warp] + g_incl - gv;
    for (int p = 0; p < nfull; ++p) units[at_full + p] = make_uint2(((uint32_t)s << 16) | (uint32_t)p, ctx);
    const int at = key == key_full ? at_full + nfull : start[key] + cnt[warp][key] + rank;
    units[at] = make_uint2(((uint32_t)s << 16) | (uint32_t)(n - 1), ctx);
  }
}

__global__ void __launch_bounds__(kPlanThreads)
    paged_decode_plan_kernel(const int32_t* __restrict__ context_lens, int num_seqs, int max_ctx, int part_tokens,
                             int sort, uint2* __restrict__ units, int* __restrict__ counters) {
  pdl_launch_dependents();
  if (sort && num_seqs <= kPlanThreads) {
    plan_sort_one_pass(context_lens, num_seqs, max_ctx, part_tokens, units, counters);
    return;
  }
  __shared__ int scratch[kPlanBuckets];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;

  if (sort) {
    // the lengths go through shared memory once (num_seqs <= kPlanSortMaxSeqs)
    __shared__ int ctx_s[kPlanSortMaxSeqs];
    for (int s = tid; s < num_seqs; s += kPlanThreads) {
      const int raw = context_lens[s];
      if (raw < 0 || raw > max_ctx) flag_error(PKV_DEV_CONTEXT_LEN);
      ctx_s[s] = clamp_ctx(raw, max_ctx);
    }
    for (int k = tid; k < kPlanBuckets; k += kPlanThreads) scratch[k] = 0;
    __syncthreads();
    if (warp != 0) return;
    pdl_wait_primary();  // the previous call's kernels may still read the list and the counters
    const unsigned below = (1u << lane) - 1u;
    const int key_full = unit_bucket(part_tokens);  // every partition but a sequence's last is full
    // pass 0 counts the units of each bucket; pass 1 places them.  A run of 32
    // sequences places its full partitions (sequence-major) then its last ones.
    for (int pass = 0; pass < 2; ++pass) {
      for (int base = 0; base < num_seqs; base += 32) {
        const int s = base + lane;
        const bool live = s < num_seqs;
        const int ctx = live ? ctx_s[s] : 0;
        const int n = live ? parts_of(ctx, part_tokens) : 0;
        const int nfull = max(n - 1, 0);
        int excl = nfull;  // exclusive scan of nfull over the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, excl, o);
          if (lane >= o) excl += v;
        }
        const int tot = __shfl_sync(0xffffffffu, excl, 31);
        excl -= nfull;
        if (pass == 1) {
          const int at = scratch[key_full] + excl;
          for (int j = 0; j < nfull; ++j) units[at + j] = make_uint2(((uint32_t)s << 16) | (uint32_t)j, ctx);
        }
        __syncwarp();
        if (lane == 0 && tot > 0) scratch[key_full] += tot;
        __syncwarp();
        const int key = live ? unit_bucket(ctx - (n - 1) * part_tokens) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, key);
        if (live && pass == 1)
          units[scratch[key] + __popc(same & below)] = make_uint2(((uint32_t)s << 16) | (uint32_t)(n - 1), ctx);
        __syncwarp();
        if (live && (same & below) == 0) scratch[key] += __popc(same);
        __syncwarp();
      }
      if (pass == 0) {  // bucket start positions, longest bucket first
        // lane l owns buckets 127-4l ... 124-4l; an exclusive scan over the lanes
        // gives each bucket the count of all longer buckets
        int c[kPlanBuckets / 32];
        int mine = 0;
#pragma unroll
        for (int j = 0; j < kPlanBuckets / 32; ++j) {
          c[j] = scratch[kPlanBuckets - 1 - (kPlanBuckets / 32) * lane - j];
          mine += c[j];
        }
        int excl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, excl, o);
          if (lane >= o) excl += v;
        }
        const int total = __shfl_sync(0xffffffffu, excl, 31);
        excl -= mine;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < kPlanBuckets / 32; ++j) {
          scratch[kPlanBuckets - 1 - (kPlanBuckets / 32) * lane - j] = excl;
          excl += c[j];
        }
        if (lane == 0) {
          counters[0] = 0;
          counters[1] = total;
        }
        __syncwarp();
      }
    }
    return;
  }

  const int per = (num_seqs + kPlanThreads - 1) / kPlanThreads;
  const int s0 = min(num_seqs, tid * per);
  const int s1 = min(num_seqs, s0 + per);
  int mine = 0;
  for (int s = s0; s < s1; ++s) {
    const int raw = context_lens[s];
    if (raw < 0 || raw > max_ctx) flag_error(PKV_DEV_CONTEXT_LEN);
    mine += parts_of(clamp_ctx(raw, max_ctx), part_tokens);
  }
  // exclusive scan over the CTA
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  pdl_wait_primary();  // the previous call's kernels may still read the list and the counters
  if (warp == 0) {
    const int w = scratch[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    scratch[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) {
      counters[0] = 0;
      counters[1] = wi;
    }
  }
  __syncthreads();
  int pos = scratch[warp] + incl - mine;
  for (int s = s0; s < s1; ++s) {
    const int ctx = clamp_ctx(context_lens[s], max_ctx);
    const int n = parts_of(ctx, part_tokens);
    for (int p = 0; p < n; ++p) units[pos++] = make_uint2(((uint32_t)s << 16) | (uint32_t)p, ctx);
  }
}

// Unit descriptor as the producer sees it.
struct UnitDesc {
  int s, h, p, t_begin, t_end, n_parts;
};

// ---------------------------------------------------------------------------
// 2. persistent decode kernel.  grid = min(#SMs x resident CTAs, units); block = 160.
// ---------------------------------------------------------------------------
template <typename T, int D, int TT, int NS>
__global__ void __launch_bounds__(kDecodeThreads) paged_decode_kernel(const DecodeParams prm) {
  using Tr = DecodeTraits<T, D, TT, NS>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* empty = full + NS;
  uint64_t* epi = empty + NS;
  int4* hdr = reinterpret_cast<int4*>(smem + Tr::kHdrOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Tr::kAbortOffset);
  float* red = reinterpret_cast<float*>(smem + Tr::kRedOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int H = prm.num_heads;
  const int PT = prm.part_tokens;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_init(epi, kConsumerWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Everything above overlaps the plan kernel; the unit list, the counters and
  // the appended cache rows are read only after it (and what precedes it) is done.
  pdl_wait_primary();

  if (warp == kConsumerWarps) {
    // ------------------------------- producer -------------------------------
    const T* kc = static_cast<const T*>(prm.k_cache);
    const T* vc = static_cast<const T*>(prm.v_cache);
    const T* qg = static_cast<const T*>(prm.q);
    const uint64_t policy = l2_evict_first();
    const int B = prm.block_size;
    const int unit_rows = min(B, TT);  // rows per bulk copy
    const int units_per_tile = TT / unit_rows;
    const long long total_units = (long long)prm.counters[1] * H;

    auto describe = [&](int u, uint2 e) {
      UnitDesc d{0, 0, 0, 0, 0, 1};
      if ((long long)u < total_units) {
        d.s = (int)(e.x >> 16);
        d.p = (int)(e.x & 0xffffu);
        d.h = u - (u / H) * H;
        const int ctx = (int)e.y;  // clamped by the plan kernel
        d.t_begin = d.p * PT;
        d.t_end = min(ctx, d.t_begin + PT);
        d.n_parts = parts_of(ctx, PT);
      }
      return d;
    };
    // CTA b starts with unit b; later units come from the counter, offset by the grid
    // size (lane 0 claims; the caller broadcasts the id when it needs it)
    auto claim = [&]() { return lane == 0 ? (int)gridDim.x + atomicAdd(&prm.counters[0], 1) : 0; };
    auto entry = [&](int u) {
      return (long long)u < total_units ? __ldcg(prm.units + u / H) : make_uint2(0u, 0u);
    };
    int u = (int)blockIdx.x;
    UnitDesc cur = describe(u, entry(u));
    int it = 0;  // stage iterations issued so far
    bool stop = false;
    while (!stop) {
      const bool done = (long long)u >= total_units;
      const int u_next_lane0 = done ? 0 : claim();  // one unit ahead
      int u_next = 0;
      uint2 e_next = make_uint2(0u, 0u);
      const int n_tok = max(0, cur.t_end - cur.t_begin);
      const int n_tiles = done ? 1 : max(1, (n_tok + TT - 1) / TT);
      const int32_t* table = prm.block_tables + (size_t)cur.s * prm.max_blocks;

      for (int i = 0; i < n_tiles; ++i, ++it) {
        const int stage = it % NS;
        // block-table entries of this tile: read before waiting for the stage
        const int tile_t0 = cur.t_begin + i * TT;
        const int u_t0 = tile_t0 + lane * unit_rows;
        const bool mine = !done && lane < units_per_tile && u_t0 < cur.t_end;
        const int phys = mine ? __ldg(table + u_t0 / B) : -1;  // u_t0 < ctx <= max_blocks * B
        if (it >= NS) {
          int ok = 1;
          if (lane == 0) ok = mbar_wait_bounded(&empty[stage], ((it / NS) - 1) & 1, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (lane == 0) {
              flag_error(PKV_DEV_WAIT_TIMEOUT);
              *abort_flag = 1;
            }
            stop = true;
            break;
          }
        }
        const int n_valid = done ? 0 : max(0, min(TT, cur.t_end - tile_t0));
        uint32_t bytes = 0;
        size_t src_off = 0;
        if (mine) {
          if (phys >= 0 && phys < prm.num_blocks) {
            const int rows = min(unit_rows, cur.t_end - u_t0);
            src_off = pool_row(phys, cur.h / prm.group, u_t0 % B, prm.num_kv_heads, B, D);
            bytes = (uint32_t)rows * Tr::kRowBytes;
          } else {
            flag_error(PKV_DEV_BLOCK_ID);
          }
        }
        uint32_t total = bytes;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        const bool load_q = (i == 0) && n_tok > 0;
        if (lane == 0) {
          const int flags = done ? kTileEnd : ((i == 0 ? kTileFirst : 0) | (i == n_tiles - 1 ? kTileLast : 0));
          hdr[stage] = make_int4(cur.s, cur.h, cur.p | (cur.n_parts << 16), n_valid | (flags << 16));
          mbar_arrive_expect_tx(&full[stage], 2u * total + (load_q ? (uint32_t)Tr::kRowBytes : 0u));
        }
        __syncwarp();
        if (bytes) {
          unsigned char* st = smem + stage * Tr::kStageBytes + lane * unit_rows * Tr::kRowBytes;
          bulk_load(st, kc + src_off, bytes, &full[stage], policy);
          bulk_load(st + Tr::kTileBytes, vc + src_off, bytes, &full[stage], policy);
        }
        if (load_q && lane == 0) {
          bulk_load(smem + Tr::kQOffset + stage * Tr::kRowBytes, qg + ((size_t)cur.s * H + cur.h) * D,
                    Tr::kRowBytes, &full[stage], policy);
        }
        if (i == 0 && !done) {  // start fetching the next unit's list entry
          u_next = __shfl_sync(0xffffffffu, u_next_lane0, 0);
          e_next = entry(u_next);
        }
      }
      if (done || stop) break;
      u = u_next;
      cur = describe(u, e_next);
    }
    pdl_launch_dependents();  // this CTA takes no more units: the merge grid may be scheduled
    // Never leave with copies in flight into this CTA's shared memory.
    if (lane == 0) {
      int no_abort = 0;
      for (int j = max(0, it - NS); j < it; ++j)
        if (!mbar_wait_bounded(&full[j % NS], (j / NS) & 1, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int grp = lane >> 3;  // token slot of this lane within the warp
  const int sub = lane & 7;   // which 16-byte chunks of a row this lane owns
  const int tok_lane = warp * 4 + grp;

  constexpr bool kNarrow = sizeof(T) == 2;  // 16-bit storage: q stays packed, q.k in mixed precision
  float qf[kNarrow ? 1 : Tr::kDimsPerLane];   // fp32 storage: q * scale_log2
  uint4 qw[Tr::kChunksPerLane];               // 16-bit storage: this lane's chunks of q
  float acc[Tr::kDimsPerLane];
#pragma unroll
  for (int k = 0; k < Tr::kDimsPerLane; ++k) acc[k] = 0.f;
#pragma unroll
  for (int k = 0; k < (kNarrow ? 1 : Tr::kDimsPerLane); ++k) qf[k] = 0.f;
#pragma unroll
  for (int c = 0; c < Tr::kChunksPerLane; ++c) qw[c] = make_uint4(0u, 0u, 0u, 0u);
  float m = -INFINITY, l = 0.f;
  int units_done = 0;

  for (int it = 0;; ++it) {
    const int stage = it % NS;
    if (!mbar_wait_bounded(&full[stage], (it / NS) & 1, abort_flag)) {
      if (lane == 0) {
        flag_error(PKV_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
      break;
    }
    const int4 hd = hdr[stage];
    const int flags = hd.w >> 16;
    const int n_valid = hd.w & 0xffff;
    if (flags & kTileEnd) break;

    if (flags & kTileFirst) {
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int k = 0; k < Tr::kDimsPerLane; ++k) acc[k] = 0.f;
      if (n_valid > 0) {
        const uint4* qrow = reinterpret_cast<const uint4*>(smem + Tr::kQOffset + stage * Tr::kRowBytes);
        if constexpr (kNarrow) {
#pragma unroll
          for (int c = 0; c < Tr::kChunksPerLane; ++c) qw[c] = qrow[c * 8 + sub];
        } else {
#pragma unroll
          for (int c = 0; c < Tr::kChunksPerLane; ++c) Elem<T>::widen(qrow[c * 8 + sub], qf + c * Tr::kPerChunk);
#pragma unroll
          for (int k = 0; k < Tr::kDimsPerLane; ++k) qf[k] *= prm.scale_log2;
        }
      }
    }

    const unsigned char* kt = smem + stage * Tr::kStageBytes;
    const unsigned char* vt = kt + Tr::kTileBytes;
    float x[Tr::kTokPerGroup];
#pragma unroll
    for (int j = 0; j < Tr::kTokPerGroup; ++j) {
      const int r = j * Tr::kGroups + tok_lane;
      float d0 = 0.f, d1 = 0.f;
      if (r < n_valid) {
        const uint4* row = reinterpret_cast<const uint4*>(kt + r * Tr::kRowBytes);
#pragma unroll
        for (int c = 0; c < Tr::kChunksPerLane; ++c) {
          if constexpr (kNarrow) {
            const uint4 kw = row[c * 8 + sub];
            MixedFma<T>::pair(qw[c].x, kw.x, d0, d1);
            MixedFma<T>::pair(qw[c].y, kw.y, d0, d1);
            MixedFma<T>::pair(qw[c].z, kw.z, d0, d1);
            MixedFma<T>::pair(qw[c].w, kw.w, d0, d1);
          } else {
            float f[Tr::kPerChunk];
            Elem<T>::widen(row[c * 8 + sub], f);
#pragma unroll
            for (int k = 0; k < Tr::kPerChunk; k += 2) {
              d0 = fmaf(qf[c * Tr::kPerChunk + k], f[k], d0);
              d1 = fmaf(qf[c * Tr::kPerChunk + k + 1], f[k + 1], d1);
            }
          }
        }
      }
      float d = d0 + d1;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      d += __shfl_xor_sync(0xffffffffu, d, 4);
      if constexpr (kNarrow) d *= prm.scale_log2;  // (fp32 storage: q carries the scale)
      x[j] = (r < n_valid) ? d : -INFINITY;
    }

    float mt = x[0];
#pragma unroll
    for (int j = 1; j < Tr::kTokPerGroup; ++j) mt = fmaxf(mt, x[j]);
    const float m_new = fmaxf(m, mt);
    if (m_new != -INFINITY) {
      const float alpha = ex2_fast(m - m_new);  // 0 while m is still -inf
      l *= alpha;
#pragma unroll
      for (int k = 0; k < Tr::kDimsPerLane; ++k) acc[k] *= alpha;
#pragma unroll
      for (int j = 0; j < Tr::kTokPerGroup; ++j) {
        const int r = j * Tr::kGroups + tok_lane;
        if (r < n_valid) {  // rows past the context are never read (they may hold NaN)
          const float pj = ex2_fast(x[j] - m_new);
          l += pj;
          const uint4* row = reinterpret_cast<const uint4*>(vt + r * Tr::kRowBytes);
#pragma unroll
          for (int c = 0; c < Tr::kChunksPerLane; ++c) {
            float f[Tr::kPerChunk];
            Elem<T>::widen(row[c * 8 + sub], f);
#pragma unroll
            for (int k = 0; k < Tr::kPerChunk; k += 2) {
              if constexpr (sizeof(T) == 2) {
                fma_x2(acc[c * Tr::kPerChunk + k], acc[c * Tr::kPerChunk + k + 1], pj, pj, f[k], f[k + 1]);
              } else {
                acc[c * Tr::kPerChunk + k] = fmaf(pj, f[k], acc[c * Tr::kPerChunk + k]);
                acc[c * Tr::kPerChunk + k + 1] = fmaf(pj, f[k + 1], acc[c * Tr::kPerChunk + k + 1]);
              }
            }
          }
        }
      }
      m = m_new;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);

    if (!(flags & kTileLast)) continue;

    // ---- unit epilogue: merge the 4 groups of the warp, then the 4 warps ----
    float mu = m, lu = l;
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {
      const float m_o = __shfl_xor_sync(0xffffffffu, mu, o);
      const float l_o = __shfl_xor_sync(0xffffffffu, lu, o);
      const float mx = fmaxf(mu, m_o);
      const float a = (mx == -INFINITY) ? 0.f : exp2f(mu - mx);
      const float b = (mx == -INFINITY) ? 0.f : exp2f(m_o - mx);
      lu = lu * a + l_o * b;
#pragma unroll
      for (int k = 0; k < Tr::kDimsPerLane; ++k) {
        const float other = __shfl_xor_sync(0xffffffffu, acc[k], o);
        acc[k] = acc[k] * a + other * b;
      }
      mu = mx;
    }
    float* rb = red + (units_done & 1) * Tr::kRedFloats;  // double-buffered across units
    float* rml = rb;                                       // [warps][2]
    float* racc = rb + 2 * kConsumerWarps;                 // [warps][D]
    if (grp == 0) {
#pragma unroll
      for (int c = 0; c < Tr::kChunksPerLane; ++c)
#pragma unroll
        for (int k = 0; k < Tr::kPerChunk; ++k)
          racc[warp * D + (c * 8 + sub) * Tr::kPerChunk + k] = acc[c * Tr::kPerChunk + k];
    }
    if (lane == 0) {
      rml[2 * warp] = mu;
      rml[2 * warp + 1] = lu;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(epi);
    if (!mbar_wait_bounded(epi, units_done & 1, abort_flag)) {
      if (lane == 0) {
        flag_error(PKV_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
      break;
    }
    ++units_done;
    const int us = hd.x, uh = hd.y, up = hd.z & 0xffff, un = hd.z >> 16;
    const size_t sh = (size_t)us * H + uh;
    const int d = threadIdx.x;  // consumer thread d finalises dimension d
    float mx = -INFINITY, L = 0.f, o = 0.f;
    if (d < D) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, rml[2 * w]);
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float sc = (mx == -INFINITY) ? 0.f : exp2f(rml[2 * w] - mx);
        L = fmaf(rml[2 * w + 1], sc, L);
        o = fmaf(racc[w * D + d], sc, o);
      }
    }
    if (d < D) {
      if (un == 1) {
        prm.out[sh * D + d] = (L > 0.f) ? o / L : 0.f;
      } else {
        const size_t ws = sh * prm.max_parts + up;
        prm.ws_acc[ws * D + d] = o;
        if (d == 0) prm.ws_ml[ws] = make_float2(mx, L);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 3. log-sum-exp merge of the partitions of each (sequence, head), one online
//    pass over the partitions with 8 of them in flight per thread.  Contexts
//    that fit one partition were finished by the decode kernel.
//    grid = (num_heads, num_seqs); block = 128, thread d owns dimension d.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128)
    paged_decode_merge_kernel(const int32_t* __restrict__ context_lens, int num_heads, int max_ctx, int part_tokens,
                              int max_parts, const float* __restrict__ ws_acc, const float2* __restrict__ ws_ml,
                              float* __restrict__ out) {
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  const int np = parts_of(clamp_ctx(__ldg(context_lens + s), max_ctx), part_tokens);
  if (np <= 1) return;  // finished by the decode kernel
  pdl_wait_primary();   // the partitions' states are complete only after the decode kernel
  const int d = threadIdx.x;
  if (d >= D) return;
  const size_t base = ((size_t)s * num_heads + h) * max_parts;
  float M = -INFINITY, L = 0.f, o = 0.f;
  for (int p0 = 0; p0 < np; p0 += 8) {
    float2 ml[8];
    float a[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = p0 + j < np;
      ml[j] = in ? __ldcg(ws_ml + base + p0 + j) : make_float2(-INFINITY, 0.f);
      a[j] = in ? __ldcg(ws_acc + (base + p0 + j) * D + d) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float mn = fmaxf(M, ml[j].x);
      if (mn == -INFINITY) continue;
      const float keep = exp2f(M - mn);     // 0 while M is -inf
      const float add = exp2f(ml[j].x - mn);
      L = L * keep + ml[j].y * add;
      o = o * keep + a[j] * add;
      M = mn;
    }
  }
  out[((size_t)s * num_heads + h) * D + d] = (L > 0.f) ? o / L : 0.f;
}

}  // namespace pkv
