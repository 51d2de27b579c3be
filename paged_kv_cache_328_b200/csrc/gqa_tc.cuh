// Paged attention for 2..64 query rows per K/V head on the 5th-generation tensor
// cores (tcgen05, sm_100a), with the roles of the operands swapped so that the
// context tokens, not the few query rows, fill the 128-lane M dimension:
//
//   S^T = K Q^T          tcgen05.mma  M=128 tokens  N=NR rows   K=D      (K tile, Q tile: shared memory)
//   P^T = 2^(S^T*scale - m_r)    eight softmax warps, thread = one token x half of the rows
//   O^T += V^T [P_hi | P_lo]^T   tcgen05.mma  M=D=128  N=2 x rows  K=128 tokens  (V and P^T: shared memory)
//
// Grouped-query decode ("PagedAttention - Efficient Memory Management for LLM
// Serving with vLLM", related-work table: grouped-query attention shares each
// K/V head among G query heads) and the verify / chunked-prefill pass with Lq
// query tokens ("vLLM PagedAttention and continuous batching", section 5) put
// R = Lq * G query rows on every K/V tile.  With R <= 64 a 128-row M tile would be
// mostly padding (the tensor-core work, the tensor-memory traffic and the
// softmax would all scale with 128 instead of R).  Here M is the tile's 128
// tokens and N is R rounded up to 16, 32 or 64 (NR): the MMAs do R/128 of the
// padded work and each softmax thread handles NR/2 values per 128 tokens.
//
// A unit is (sequence s, K/V head kvh, row tile rt, partition p) from the plan
// kernel's list; row r of a tile is query token rt*Tq + r/G, query head kvh*G + r%G.
//
// Softmax across lanes.  A row's values sit in one column of 128 lanes, so its
// maximum and sum are cross-thread reductions.  The rows are split between two
// groups of four warps (rows [0, NR/2) and [NR/2, NR)); a group owns its rows'
// softmax state outright, so the groups never wait for each other.  Within a
// group the maximum is reduced only on a unit's first tile (it becomes the row's
// reference m_r); on later tiles each thread forms t = x*scale - m_r with one
// FMA and the group checks whether any t exceeds 8 (log2 units).  Only then does
// it reduce the tile's row maxima, raise m_r, shift t and rescale O (rare: P
// values stay below 2^8, so fp32 sums are exact to rounding either way).  The
// row sums l_r are kept per thread (one partial sum per row for the tokens this
// thread has seen) and reduced once, at the unit's end.  P is split into its
// 16-bit rounding and the 16-bit rounding of the remainder, placed side by side
// in N, so one MMA accumulates both parts: O_r = O[hi column r] + O[lo column r].
// Weights single-rounded to 16 bits would exceed the 2e-3 error bound.
//
// Warp roles (one CTA per SM, persistent over the unit list):
//   warp 0     producer: the unit's query tile (4-D TMA box, double-buffered) and
//              the 128-token K/V tiles (2-D TMA boxes per (block, K/V head) run,
//              128-byte swizzle, kNS stages);
//   warp 1     allocates / frees the tensor memory; its lane 0 issues the S products;
//   warps 2-9  softmax and epilogue, group (w - 2) / 4; warp w owns tensor-memory
//              lanes 32*(w%4) ... (tokens of S^T, dimensions of O^T);
//   warp 10    its lane 0 issues the P V products;
//   warp 11    V producer: the V half of each K/V tile, published by warp 0.
// P^T of a tile is written over the tile's K slabs (dead once S^T is computed).
// Each group exchanges reduction partials through shared memory and its own
// mbarrier (bounded waits: a failing wait cannot strand the other warps).
#pragma once

#include "multi_query_tc.cuh"

namespace pkv {

constexpr int kKtTile = 128;         // tokens per K/V tile = M of S^T = K of O^T
constexpr int kKtSoftmaxWarps = 8;   // two groups of four: warps 2-9
constexpr int kKtPvWarp = 2 + kKtSoftmaxWarps;  // issues the P V products
constexpr int kKtVWarp = 3 + kKtSoftmaxWarps;   // issues the V tiles' TMA loads
constexpr int kKtThreads = (4 + kKtSoftmaxWarps) * 32;
constexpr float kKtRescaleLog2 = 8.0f;
// A softmax group's final output rows leave through one bulk copy per run of
// consecutive rows (the rows of one query token are G consecutive query heads)
// when that takes at most this many copies; otherwise, and for the strided rows
// of partition states, the threads store them directly.  Measured on B200 (batch
// 256, attention call): bulk copies ahead by 3-4 % with one or two runs (G = 8,
// 32) and by ~1 % with two to four (G = 4 and 4 tokens, G = 2 and 8); direct
// stores ahead by 2 % with eight runs (G = 1, 8 tokens), 7 % with sixteen (G = 1,
// 32 tokens) and 11 % on 512-token partitions (G = 32).
constexpr int kKtMaxBulkRuns = 4;

// Instruction descriptor for kind::f16 with fp32 accumulation and either operand
// MN-major (bit 15: A, bit 16: B).
template <typename T>
__host__ __device__ constexpr uint32_t umma_idesc_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (TcFormat<T>::kCode << 7) | (TcFormat<T>::kCode << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t tmem_alloc_cols(uint32_t n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}

template <int NR>
struct KtTraits {
  static_assert(NR == 16 || NR == 32 || NR == 64, "row tile of 16, 32 or 64");
  static constexpr int D = 128;
  static constexpr int NH = NR / 2;                    // rows per softmax group
  // P^T row: hi at column 0, lo at column kPW / 2; kPW / 64 slabs of 128 rows
  static constexpr int kPW = NR <= 32 ? 64 : 2 * NR;
  static constexpr int kNS = 3;                        // K/V stages of 64 KB
  // query tiles: two (the next unit's loads while this one runs), one at 64 rows
  // (shared memory), loaded as soon as the previous unit's last S product is done
  static constexpr int kNQ = NR <= 32 ? 2 : 1;
  static constexpr int kSlab = kKtTile * 128;          // 128 rows x 64 columns, 16-bit: 16 KB
  static constexpr int kStageBytes = 4 * kSlab;        // K (2 slabs), V (2 slabs)
  static constexpr int kQSlab = NR * 128;
  static constexpr int kQBytes = 2 * kQSlab;
  static constexpr int kQOffset = kNS * kStageBytes;
  static constexpr int kHdrOffset = kQOffset + kNQ * kQBytes;  // after the query buffers
  static constexpr int kRowsOffset = kHdrOffset + kNS * 32;  // [NS][32] pool rows of a tile's runs (-1: none)
  static constexpr int kRedOffset = kRowsOffset + kNS * 128;  // [group][parity][NH][4 warps] floats
  static constexpr int kWarpOffset = kRedOffset + 2 * 2 * NH * 4 * 4;  // [softmax warp][mref, tmp, 1/l: NH each]
  static constexpr int kVoteOffset = kWarpOffset + kKtSoftmaxWarps * 3 * NH * 4;  // [group][parity][4] ints
  static constexpr int kBarOffset = kVoteOffset + 2 * 2 * 4 * 4;
  // full[NS], empty[NS], q_full[2], q_empty[2], s_full[2], s_free[2], p_full, pv_done, grp[2], drain[2], meta[NS]
  static constexpr int kNumBars = 3 * kNS + 14;
  static constexpr int kTmemSlotOffset = kBarOffset + kNumBars * 8;
  static constexpr int kAbortOffset = kTmemSlotOffset + 8;
  static constexpr int kSmemBytes = kAbortOffset + 8;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // the base is rounded up to 1024 bytes
  static constexpr uint32_t kOCol = 2 * NR;             // S^T buffer b at columns b * NR
  static constexpr uint32_t kTmemCols = tmem_alloc_cols(2 * NR + kPW);
  static_assert(kQOffset % 1024 == 0 && kQBytes % 1024 == 0, "swizzle atoms are 1024-byte aligned");
  static_assert(kPW / 64 <= 2, "P^T fits the K slabs of a stage");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA");
};

// Non-blocking test of a barrier phase (mbarrier.test_wait never suspends the thread).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Spin on a phase expected to complete within a short while (the softmax group's
// own barrier): test_wait reacts sooner than a suspending try_wait.  Bounded like
// mbar_wait_bounded.
__device__ __forceinline__ bool mbar_spin_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}

// Bulk (copy-engine) store of `bytes` contiguous bytes from this CTA's shared
// memory to global memory, tracked by the issuing thread's bulk async-group.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_addr(ssrc)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The shared-memory sources of this thread's bulk stores may be overwritten.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// This thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- cross-warp reductions of one softmax group ------------------------------

// One level of a butterfly reduce-scatter over the warp: of N values, a lane keeps
// the upper half if (lane & off), else the lower half, combined with its partner's.
template <int N, bool kMax>
__device__ __forceinline__ void rs_level(float* v, int lane, int off) {
  const bool up = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, off);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}

// Reduces v[0..N) (max or sum) over the group's 128 threads into out[0..N), this
// warp's copy of the result in shared memory (each warp writes its own copy, so
// it reads it back after __syncwarp alone).  Within a warp a reduce-scatter
// leaves each lane the warp's partial for max(N/32, 1) rows (N < 32: 32/N lanes
// share a row); the group's four warps meet in red[k & 1] ([row][warp]) after
// phase k of the group's barrier.  Returns false if that wait failed (abort or
// timeout).
// Reduce-scatter of 32 values over the warp: lane l returns the warp's partial of value l.
template <bool kMax>
__device__ __forceinline__ float warp_rs32(const float* v, int lane) {
  float w[16];
  const bool up = (lane & 16) != 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float send = up ? v[i] : v[i + 16];
    const float keep = up ? v[i + 16] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
    w[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
  rs_level<16, kMax>(w, lane, 8);
  rs_level<8, kMax>(w, lane, 4);
  rs_level<4, kMax>(w, lane, 2);
  rs_level<2, kMax>(w, lane, 1);
  return w[0];
}

template <int N, bool kMax>
__device__ __forceinline__ bool group_reduce(const float (&v)[N], float* red, float* out, uint64_t* grp, int& k,
                                             int q4, int lane, volatile int* abort_flag) {
  static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 rows per group");
  float* buf = red + (k & 1) * N * 4;
  if constexpr (N == 32) {
    buf[lane * 4 + q4] = warp_rs32<kMax>(v, lane);  // lane l holds row l
  } else {
    float w[N / 2];
    {
      const bool up = (lane & 16) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float send = up ? v[i] : v[i + N / 2];
        const float keep = up ? v[i + N / 2] : v[i];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
        w[i] = kMax ? fmaxf(keep, recv) : keep + recv;
      }
    }
    rs_level<N / 2, kMax>(w, lane, 8);
    if constexpr (N >= 8) rs_level<N / 4, kMax>(w, lane, 4);
    if constexpr (N >= 16) rs_level<N / 8, kMax>(w, lane, 2);
    // lanes that hold the same row (N < 32) finish with a butterfly all-reduce
    {
      const float o = __shfl_xor_sync(0xffffffffu, w[0], 1);
      w[0] = kMax ? fmaxf(w[0], o) : w[0] + o;
    }
    if constexpr (N <= 8) {
      const float o = __shfl_xor_sync(0xffffffffu, w[0], 2);
      w[0] = kMax ? fmaxf(w[0], o) : w[0] + o;
    }
    constexpr int kShare = 32 / N;  // lanes per row
    if (lane % kShare == 0) buf[(lane / kShare) * 4 + q4] = w[0];
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(grp);
  const bool ok = __all_sync(0xffffffffu, mbar_spin_bounded(grp, (uint32_t)(k & 1), abort_flag));
  ++k;
  if (!ok) return false;
  if (lane < N) {
    const float4 f = reinterpret_cast<const float4*>(buf)[lane];
    out[lane] = kMax ? fmaxf(fmaxf(f.x, f.y), fmaxf(f.z, f.w)) : (f.x + f.y) + (f.z + f.w);
  }
  __syncwarp();
  return true;
}

// Barrier of the group's four warps (same barrier as its reductions).
__device__ __forceinline__ bool group_sync(uint64_t* grp, int& k, int lane, volatile int* abort_flag) {
  __syncwarp();
  if (lane == 0) mbar_arrive(grp);
  const bool ok = __all_sync(0xffffffffu, mbar_spin_bounded(grp, (uint32_t)(k & 1), abort_flag));
  ++k;
  return ok;
}

// OR of one predicate over the group's 128 threads (same barrier as its reductions).
__device__ __forceinline__ bool group_any(bool pred, int* vote, uint64_t* grp, int& k, int q4, int lane,
                                          volatile int* abort_flag, bool& ok_out) {
  const bool any = __any_sync(0xffffffffu, pred);
  int* buf = vote + (k & 1) * 4;
  if (lane == 0) {
    buf[q4] = any ? 1 : 0;
    mbar_arrive(grp);
  }
  const bool ok = __all_sync(0xffffffffu, mbar_spin_bounded(grp, (uint32_t)(k & 1), abort_flag));
  ++k;
  ok_out = ok;
  if (!ok) return false;
  const int4 b = *reinterpret_cast<const int4*>(buf);
  return (b.x | b.y | b.z | b.w) != 0;
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// Redefine 8 registers after a tcgen05.wait::ld so that no use is scheduled above it.
__device__ __forceinline__ void tmem_pin8(uint32_t* r) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}

// tcgen05.ld of N consecutive 32-bit columns of this thread's lane (N = 8, 16, 32).
template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&x)[N]) {
  uint32_t v[N];
#pragma unroll
  for (int c = 0; c < N / 8; ++c) tmem_ld8(taddr + 8 * c, v + 8 * c);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < N / 8; ++c) tmem_pin8(v + 8 * c);
#pragma unroll
  for (int i = 0; i < N; ++i) x[i] = __uint_as_float(v[i]);
}

// grid = min(#SMs, units); block = kKtThreads; one CTA per SM (shared memory).
template <typename T, int NR>
__global__ void __launch_bounds__(kKtThreads, 1) paged_gqa_tc_kernel(const __grid_constant__ TcParams prm) {
  using Tr = KtTraits<NR>;
  constexpr int D = Tr::D;
  constexpr int NS = Tr::kNS;
  constexpr int NH = Tr::NH;
  constexpr int NQ = Tr::kNQ;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;  // [2]
  uint64_t* q_empty = q_full + 2;    // [2]
  uint64_t* s_full = q_full + 4;     // [2]
  uint64_t* s_free = q_full + 6;     // [2]
  uint64_t* p_full = q_full + 8;
  uint64_t* pv_done = q_full + 9;
  uint64_t* grp = q_full + 10;       // [2]: one per softmax group
  uint64_t* drain = q_full + 12;     // [2]: one per MMA issuer
  uint64_t* meta = q_full + 14;      // [NS]: a tile's header and pool rows are published
  int* run_rows = reinterpret_cast<int*>(smem + Tr::kRowsOffset);
  int4* hdr = reinterpret_cast<int4*>(smem + Tr::kHdrOffset);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::kTmemSlotOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Tr::kAbortOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Hkv = prm.num_kv_heads;
  const int G = prm.group;
  const int Tq = prm.tq_per_tile;
  const int RT = prm.row_tiles;
  const int PT = prm.part_tokens;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 3);  // the P V commit, then one arrival per softmax group
      mbar_init(&meta[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kKtSoftmaxWarps);
      mbar_init(&grp[i], 4);
    }
    mbar_init(p_full, kKtSoftmaxWarps);
    mbar_init(pv_done, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // query rows that no TMA box covers read as zero (their logits are masked in any case)
  for (int i = threadIdx.x; i < Tr::kNQ * Tr::kQBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + Tr::kQOffset)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(Tr::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_primary();

  const int per_sp = Hkv * RT;  // units per (sequence, partition)
  const long long total_units = (long long)prm.counters[1] * per_sp;

  if (warp == 0) {
    // ------------------------------- producer -------------------------------
    const uint64_t policy = l2_evict_first();
    const int B = prm.block_size;
    const int unit_rows = min(B, kKtTile);
    const int units_per_tile = kKtTile / unit_rows;
    const uint32_t run_bytes = (uint32_t)(unit_rows * 128);
    const uint32_t q_bytes = (uint32_t)(2 * 128 * G * Tq);

    auto describe = [&](int u, uint2 e) {
      TcUnit d{0, 0, 0, 0, 0, 0, 1, 0};
      if ((long long)u < total_units) {
        d.s = (int)(e.x >> 16);
        d.p = (int)(e.x & 0xffffu);
        const int rem = u - (u / per_sp) * per_sp;
        d.kvh = rem / RT;
        d.rt = rem - d.kvh * RT;
        d.ctx = (int)e.y;
        d.t_begin = d.p * PT;
        d.t_end = min(d.ctx, d.t_begin + PT);
        d.n_parts = parts_of(d.ctx, PT);
      }
      return d;
    };
    auto claim = [&]() { return lane == 0 ? (int)gridDim.x + atomicAdd(&prm.counters[0], 1) : 0; };
    auto entry = [&](int u) {
      return (long long)u < total_units ? __ldcg(prm.units + u / per_sp) : make_uint2(0u, 0u);
    };

    // pool blocks of a tile's runs: lane l < units_per_tile reads the block of run l
    auto run_blocks = [&](const TcUnit& d, int tile_t0) {
      const int u_t0 = tile_t0 + lane * unit_rows;
      return (lane < units_per_tile && u_t0 < d.t_end)
                 ? __ldg(prm.block_tables + (size_t)d.s * prm.max_blocks + u_t0 / B)  // u_t0 < ctx <= max_blocks * B
                 : -1;
    };

    int u = (int)blockIdx.x;
    TcUnit cur = describe(u, entry(u));
    // block-table entries are read one tile ahead (across unit boundaries too), so
    // that their latency hides behind the previous tile's stage wait and loads
    int phys_nx = run_blocks(cur, cur.t_begin);
    int it = 0;        // tiles issued
    // Query tiles (lane 0's bookkeeping): unit n's goes to buffer n % NQ once the S
    // products of unit n - NQ are done.  A unit's tile is owed as soon as the unit
    // is known (at the previous unit's last tile) and issued as soon as its buffer
    // is free, also while this warp waits for a stage, so the K/V tiles never wait
    // for it.  With one buffer (NQ = 1) only the first unit's is issued here; the
    // S issuer issues each next one the moment the last S product frees the buffer.
    int nu = 0;        // query tiles issued
    int owed = 0;      // query tiles owed up to this count
    TcUnit q_unit = cur;
    auto q_ready = [&]() {
      return nu < NQ || mbar_test(&q_empty[nu % NQ], (uint32_t)(((nu / NQ) - 1) & 1));
    };
    auto q_issue = [&]() {  // lane 0
      const int qb = nu % NQ;
      mbar_arrive_expect_tx(&q_full[qb], q_bytes);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        tma_load_4d(smem + Tr::kQOffset + qb * Tr::kQBytes + hf * Tr::kQSlab, &prm.tmap_q, hf * 64,
                    q_unit.kvh * G, q_unit.rt * Tq, q_unit.s, &q_full[qb], policy);
      ++nu;
    };
    // lane 0: wait (bounded) until the owed query tile can be issued, and issue it
    auto q_settle = [&]() {
      if (nu == owed) return true;
      const long long t0 = clock64();
      while (!q_ready()) {
        if (*abort_flag || clock64() - t0 > kWaitLimitCycles) return false;
      }
      q_issue();
      return true;
    };
    // owe unit d's query tile (the previous one is issued first); false on a timeout
    auto q_owe = [&](const TcUnit& d) {
      int ok = 1;
      if (lane == 0) {
        ok = q_settle();
        if (ok) {
          q_unit = d;
          ++owed;
          if (q_ready()) q_issue();
        }
      }
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    bool stop = false;
    if ((long long)u < total_units && !q_owe(cur)) stop = true;
    while (!stop) {
      const bool done = (long long)u >= total_units;
      const int u_next_lane0 = done ? 0 : claim();
      int u_next = 0;
      uint2 e_next = make_uint2(0u, 0u);
      TcUnit nxt{0, 0, 0, 0, 0, 0, 1, 0};
      const int n_tok = max(0, cur.t_end - cur.t_begin);
      const int n_tiles = done ? 1 : max(1, (n_tok + kKtTile - 1) / kKtTile);

      for (int i = 0; i < n_tiles; ++i, ++it) {
        const int stage = it % NS;
        const int tile_t0 = cur.t_begin + i * kKtTile;
        const int u_t0 = tile_t0 + lane * unit_rows;
        const bool mine = !done && lane < units_per_tile && u_t0 < cur.t_end;
        const int phys = phys_nx;
        // the next tile's blocks: this unit's next tile, or the next unit's first
        // (its list entry was read at this unit's first tile; a one-tile unit reads
        // them at the end of its tile)
        bool next_known = false;
        if (!done) {
          if (i + 1 < n_tiles) {
            phys_nx = run_blocks(cur, tile_t0 + kKtTile);
          } else if (i > 0) {
            nxt = describe(u_next, e_next);
            phys_nx = run_blocks(nxt, nxt.t_begin);
            next_known = true;
          }
        }
        if (it >= NS) {
          int ok = 1;
          if (lane == 0) {
            const uint32_t par = ((it / NS) - 1) & 1;
            if (nu == owed) {
              ok = mbar_wait_bounded(&empty[stage], par, abort_flag);
            } else {
              // poll: the owed query tile goes out as soon as its buffer is free
              const long long t0 = clock64();
              while (!mbar_test(&empty[stage], par)) {
                if (nu < owed && q_ready()) q_issue();
                if (*abort_flag || clock64() - t0 > kWaitLimitCycles) {
                  ok = 0;
                  break;
                }
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            stop = true;
            break;
          }
        }
        const int n_valid = done ? 0 : max(0, min(kKtTile, cur.t_end - tile_t0));
        bool load = false;
        if (mine) {
          if (phys >= 0 && phys < prm.num_blocks)
            load = true;
          else
            flag_error(PKV_DEV_BLOCK_ID);
        }
        const unsigned loads = __ballot_sync(0xffffffffu, load);
        const int y = load ? (phys * Hkv + cur.kvh) * B + (u_t0 % B) : -1;
        // publish the tile (header, pool row of each run) for the V producer, arm the
        // stage's barrier with the bytes of both halves, then load the K half
        run_rows[stage * 32 + lane] = y;
        if (lane == 0) {
          const int flags = done ? kTileEnd : ((i == 0 ? kTileFirst : 0) | (i == n_tiles - 1 ? kTileLast : 0));
          hdr[2 * stage] = make_int4(cur.s, cur.kvh | (cur.rt << 16), cur.p | (cur.n_parts << 16),
                                     n_valid | (flags << 16));
          hdr[2 * stage + 1] = make_int4(tile_t0, cur.ctx, 0, 0);
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], (uint32_t)__popc(loads) * 4u * run_bytes);
          mbar_arrive(&meta[stage]);
        }
        if (load) {
          unsigned char* kt = smem + stage * Tr::kStageBytes + lane * unit_rows * 128;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) tma_load_2d(kt + hf * Tr::kSlab, &prm.tmap_k, hf * 64, y, &full[stage], policy);
        }
        if (i == 0 && !done) {
          u_next = __shfl_sync(0xffffffffu, u_next_lane0, 0);
          e_next = entry(u_next);
          if (n_tiles == 1) {
            nxt = describe(u_next, e_next);
            phys_nx = run_blocks(nxt, nxt.t_begin);
            next_known = true;
          }
        }
        if (NQ > 1 && next_known && (long long)u_next < total_units && !q_owe(nxt)) {
          stop = true;
          break;
        }
      }
      if (done || stop) break;
      u = u_next;
      cur = nxt;
    }
    if (stop && lane == 0) {
      flag_error(PKV_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    // the last unit's query tile, if still owed
    if (lane == 0 && !stop && !q_settle()) {
      flag_error(PKV_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
    pdl_launch_dependents();
    // never leave with copies in flight into this CTA's shared memory
    if (lane == 0) {
      int no_abort = 0;
      for (int j = max(0, it - NS); j < it; ++j)
        if (!mbar_wait_bounded(&full[j % NS], (j / NS) & 1, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
      // (with one query buffer the S issuer also loads it, and drains it)
      if (NQ > 1)
        for (int j = max(0, nu - NQ); j < nu; ++j)
          if (!mbar_wait_bounded(&q_full[j % NQ], (j / NQ) & 1, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
  } else if (warp == kKtVWarp) {
    // ------------------------------ V producer ------------------------------
    // Follows the K producer tile by tile: once a tile is published (meta), each
    // run's V rows go to the stage's V slabs, completing on the same barrier.
    const uint64_t policy = l2_evict_first();
    const int unit_rows = min(prm.block_size, kKtTile);
    for (int t = 0;; ++t) {
      const int stage = t % NS;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&meta[stage], (t / NS) & 1, abort_flag))) {
        if (lane == 0) {
          flag_error(PKV_DEV_WAIT_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      if ((hdr[2 * stage].w >> 16) & kTileEnd) break;
      const int y = run_rows[stage * 32 + lane];
      if (y >= 0) {
        unsigned char* vt = smem + stage * Tr::kStageBytes + 2 * Tr::kSlab + lane * unit_rows * 128;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) tma_load_2d(vt + hf * Tr::kSlab, &prm.tmap_v, hf * 64, y, &full[stage], policy);
      }
    }
  } else if (warp == 1 || warp == kKtPvWarp) {
    // ----------------------------- MMA issuers -----------------------------
    // Warp 1 issues the S products, warp kKtPvWarp the P V products, each in tile
    // order with its own commits, so that neither waits behind the other's
    // issue.  Shared-memory descriptors are formed once; an MMA adds a constant
    // offset to the start-address field (16-byte units; every operand lies below
    // 256 KB).
    if (lane == 0) {
      bool ok = true;
      if (warp == 1) {
        constexpr uint32_t kIdescS = umma_idesc_ab<T>(kKtTile, NR, false, false);
        const uint64_t desc_k0 = umma_desc_sw128(smem_addr(smem), 16, 1024);
        const uint64_t desc_q0 = umma_desc_sw128(smem_addr(smem + Tr::kQOffset), 16, 1024);
        const uint64_t policy = l2_evict_first();
        int nq = 0;  // query tiles consumed
        // NQ = 1: query tiles issued (the producer issues the first unit's)
        int nq_issued = (long long)blockIdx.x < total_units ? 1 : 0;
        for (int t = 0;; ++t) {
          const int stage = t % NS;
          if (!mbar_wait_bounded(&full[stage], (t / NS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int flags = hdr[2 * stage].w >> 16;
          if (flags & kTileEnd) break;
          if (flags & kTileFirst) {
            if (!mbar_wait_bounded(&q_full[nq % NQ], (nq / NQ) & 1, abort_flag)) {
              ok = false;
              break;
            }
            ++nq;
          }
          const int qb = (nq - 1) % NQ;
          const int sb = t & 1;
          if (t >= 2 && !mbar_wait_bounded(&s_free[sb], ((t >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_k0 + (uint64_t)((stage * Tr::kStageBytes) >> 4);
          const uint64_t b0 = desc_q0 + (uint64_t)((qb * Tr::kQBytes) >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            // 16 columns = 32 bytes inside a 64-column slab
            const uint32_t ka = (uint32_t)((k >> 2) * Tr::kSlab + (k & 3) * 32) >> 4;
            const uint32_t kb = (uint32_t)((k >> 2) * Tr::kQSlab + (k & 3) * 32) >> 4;
            umma_f16(tmem_base + (uint32_t)(sb * NR), a0 + ka, b0 + kb, kIdescS, k > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          if (flags & kTileLast) {
            umma_commit(&q_empty[qb]);
            if constexpr (NQ == 1) {
              // The one query buffer is free once this product is done: load the
              // next unit's rows (the next tile, published by the producer, opens it)
              // right away rather than when the producer next looks.
              const int tn = t + 1, sn = tn % NS;
              if (!mbar_wait_bounded(&q_empty[0], (uint32_t)((nq - 1) & 1), abort_flag) ||
                  !mbar_wait_bounded(&meta[sn], (uint32_t)((tn / NS) & 1), abort_flag)) {
                ok = false;
                break;
              }
              const int4 hn = hdr[2 * sn];
              if (!((hn.w >> 16) & kTileEnd)) {
                mbar_arrive_expect_tx(&q_full[0], (uint32_t)(2 * 128 * G * Tq));
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                  tma_load_4d(smem + Tr::kQOffset + hf * Tr::kQSlab, &prm.tmap_q, hf * 64, (hn.y & 0xffff) * G,
                              (hn.y >> 16) * Tq, hn.x, &q_full[0], policy);
                ++nq_issued;
              }
            }
          }
        }
        if (NQ == 1 && nq_issued > nq) {
          // never leave with a query tile in flight into this CTA's shared memory
          int no_abort = 0;
          if (!mbar_wait_bounded(&q_full[0], (uint32_t)((nq_issued - 1) & 1), &no_abort)) ok = false;
        }
      } else {
        constexpr uint32_t kIdescO = umma_idesc_ab<T>(D, Tr::kPW, true, true);
        const uint64_t desc_v0 = umma_desc_sw128(smem_addr(smem + 2 * Tr::kSlab), Tr::kSlab, 1024);  // V (A)
        const uint64_t desc_p0 = umma_desc_sw128(smem_addr(smem), Tr::kSlab, 1024);  // P^T over the K slabs (B)
        for (int t = 0;; ++t) {
          const int stage = t % NS;
          // the stage is released by this warp's commit below, so its header stays valid
          if (!mbar_wait_bounded(&full[stage], (t / NS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int flags = hdr[2 * stage].w >> 16;
          if (flags & kTileEnd) break;
          if (!mbar_wait_bounded(p_full, (uint32_t)(t & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc_v0 + (uint64_t)((stage * Tr::kStageBytes) >> 4);
          const uint64_t b0 = desc_p0 + (uint64_t)((stage * Tr::kStageBytes) >> 4);
          const bool fp = flags & kTileFirst;
          // 16 tokens per step (16 rows x 128 bytes); steps wholly past the tile's
          // valid tokens add nothing (their weights are 0) and are skipped; an
          // empty tile still runs one step (zero weights) so that O starts at 0
          const int steps = max(1, ((hdr[2 * stage].w & 0xffff) + 15) / 16);
#pragma unroll
          for (int k = 0; k < kKtTile / 16; ++k)
            if (k < steps)
              umma_f16(tmem_base + Tr::kOCol, a0 + (uint64_t)(k * (2048 >> 4)), b0 + (uint64_t)(k * (2048 >> 4)),
                       kIdescO, (fp && k == 0) ? 0u : 1u);
          umma_commit(&empty[stage]);
          umma_commit(pv_done);
          // a unit's last stage also holds its output rows until they are stored:
          // there each softmax group releases it; elsewhere this thread does
          if (!(flags & kTileLast)) {
            mbar_arrive(&empty[stage]);
            mbar_arrive(&empty[stage]);
          }
        }
      }
      if (!ok) {
        flag_error(PKV_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA this thread issued must be complete before the tensor memory is freed
      uint64_t* my_drain = warp == 1 ? drain : drain + 1;
      umma_commit(my_drain);
      int no_abort = 0;
      if (!mbar_wait_bounded(my_drain, 0, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // --------------------------- softmax / epilogue ---------------------------
    const int sg = (warp - 2) >> 2;    // softmax group: rows [sg * NH, sg * NH + NH)
    const int q4 = warp & 3;           // tensor-memory lane quarter of this warp
    const int tl = q4 * 32 + lane;     // token of S^T and dimension of O^T owned by this thread
    const int r0 = sg * NH;            // first row of this group
    const uint32_t tlane = tmem_base + ((uint32_t)(q4 * 32) << 16);
    const int Lq = prm.q_len;
    const float scale = prm.scale_log2;
    float* red = reinterpret_cast<float*>(smem + Tr::kRedOffset) + sg * 2 * NH * 4;
    int* vote = reinterpret_cast<int*>(smem + Tr::kVoteOffset) + sg * 2 * 4;
    uint64_t* my_grp = &grp[sg];
    // this warp's copies of its rows' reference maxima and of a per-row scratch
    // (the excess of a tile's maxima over the references, then the row sums)
    float* mref = reinterpret_cast<float*>(smem + Tr::kWarpOffset) + (warp - 2) * 3 * NH;
    float* tmp = mref + NH;
    float* inv = tmp + NH;
    const float4* mref4 = reinterpret_cast<const float4*>(mref);
    const float4* tmp4 = reinterpret_cast<const float4*>(tmp);
    float lpart[NH];  // this thread's share of each row's sum of weights
#pragma unroll
    for (int r = 0; r < NH; ++r) lpart[r] = 0.f;
    int gk = 0;       // group barrier phases used
    int pv_seen = 0;  // P V products observed complete (pv_done phases waited in order)
    bool failed = false;
    // every lane waits (each observes the phase itself); the outcome is made uniform
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag));
    };
    auto wait_pv = [&](int tp) {
      if (tp < pv_seen) return true;
      if (!wait_all(pv_done, (uint32_t)(tp & 1))) return false;
      pv_seen = tp + 1;
      return true;
    };

    for (int j = 0;; ++j) {
      const int stage = j % NS;
      if (!wait_all(&full[stage], (j / NS) & 1)) {
        failed = true;
        break;
      }
      const int4 hd = hdr[2 * stage];
      const int4 hd2 = hdr[2 * stage + 1];
      const int flags = hd.w >> 16;
      const int n_valid = hd.w & 0xffff;
      if (flags & kTileEnd) break;
      const int sb = j & 1;
      if (!wait_all(&s_full[sb], (j >> 1) & 1)) {
        failed = true;
        break;
      }
      tc_fence_after();
      float x[NH];
      tmem_ld_row<NH>(tlane + (uint32_t)(sb * NR + r0), x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      // rows r in [r_lo, r_hi) see this thread's token: query token tq sees
      // positions < ctx - Lq + tq + 1, and only tokens tq < Lq exist
      const int t0 = hd2.x, ctx = hd2.y;
      const int rt = hd.y >> 16;
      const int j0 = t0 + tl - ctx + Lq - rt * Tq;  // first local query token that sees it
      const int r_lo = min(max(j0, 0), Tq) * G;
      const int r_hi = tl < n_valid ? min(Tq, Lq - rt * Tq) * G : 0;
      // every row of the group sees every token of the warp: no masking needed
      const bool open = __all_sync(0xffffffffu, r_lo <= r0 && r_hi >= r0 + NH);

      // rows this thread's token is hidden from get t = -inf (after the scaling,
      // so that a row no token sees, whose m_r is -inf, cannot turn into +inf)
      auto mask_hidden = [&]() {
        if (!open) {
          const int lo = r_lo - r0, hi = r_hi - r0;  // visible rows of this group: [lo, hi)
#pragma unroll
          for (int r = 0; r < NH; ++r) x[r] = (r >= lo && r < hi) ? x[r] : -INFINITY;
        }
      };
      // t = x * scale - m_r (log2 units, -inf where masked)
      if (flags & kTileFirst) {
        // the unit's reference maxima: this tile's row maxima
#pragma unroll
        for (int r = 0; r < NH; ++r) x[r] *= scale;
        mask_hidden();
        if (!group_reduce<NH, true>(x, red, mref, my_grp, gk, q4, lane, abort_flag)) {
          failed = true;
          break;
        }
#pragma unroll
        for (int c = 0; c < NH / 4; ++c) {
          const float4 m = mref4[c];
          const float mm[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 4 * c + i;
            x[r] = x[r] == -INFINITY ? -INFINITY : x[r] - mm[i];  // a row no token sees keeps m_r = -inf
            lpart[r] = 0.f;
          }
        }
      } else {
        // a row that some token sees has a finite m_r (visibility is a prefix of the partition)
#pragma unroll
        for (int c = 0; c < NH / 4; ++c) {
          // x * scale - m_r, two rows per packed fp32 FMA (each rounded as fmaf)
          const float4 m = mref4[c];
          float t0 = -m.x, t1 = -m.y, t2 = -m.z, t3 = -m.w;
          fma_x2(t0, t1, x[4 * c], x[4 * c + 1], scale, scale);
          fma_x2(t2, t3, x[4 * c + 2], x[4 * c + 3], scale, scale);
          x[4 * c] = t0;
          x[4 * c + 1] = t1;
          x[4 * c + 2] = t2;
          x[4 * c + 3] = t3;
        }
        mask_hidden();
        float tmax = -INFINITY;
#pragma unroll
        for (int r = 0; r < NH; ++r) tmax = fmaxf(tmax, x[r]);
        bool ok = true;
        const bool need = group_any(tmax > kKtRescaleLog2, vote, my_grp, gk, q4, lane, abort_flag, ok);
        if (!ok) {
          failed = true;
          break;
        }
        if (need) {
          // raise each row's reference by its tile maximum's excess d >= 0: t -= d,
          // and the row's earlier weights (l, O) scale by 2^-d
          if (!group_reduce<NH, true>(x, red, tmp, my_grp, gk, q4, lane, abort_flag)) {
            failed = true;
            break;
          }
          if (lane < NH) {
            const float d = fmaxf(tmp[lane], 0.f);  // -inf (no visible token) gives 0
            tmp[lane] = d;
            mref[lane] += d;
          }
          __syncwarp();
#pragma unroll
          for (int c = 0; c < NH / 4; ++c) {
            const float4 dd = tmp4[c];
            const float dv[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 4 * c + i;
              x[r] -= dv[i];
              lpart[r] *= ex2_fast(-dv[i]);
            }
          }
          // O holds every product of this unit issued so far: all must be complete
          if (!wait_pv(j - 1)) {
            failed = true;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int c = 0; c < NH / 8; ++c) {
              const uint32_t col = tlane + Tr::kOCol + (uint32_t)(part * (Tr::kPW / 2) + r0 + 8 * c);
              uint32_t v[8];
              tmem_ld8(col, v);
              tmem_wait_ld();
              tmem_pin8(v);
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * ex2_fast(-tmp[8 * c + i]));
              tmem_st8(col, v);
            }
          }
          tmem_wait_st();
        }
      }

      {
        // this thread's row of the MN-major P^T operand, columns of the group's
        // rows: p = 2^t split into high and low 16-bit parts, 8 columns (16 bytes)
        // per chunk, the chunk index XORed with tl mod 8 (128-byte swizzle); hi at
        // column r, lo at column kPW / 2 + r.  It goes over the stage's K slabs:
        // S^T of this tile, their only reader, is complete (s_full).
        unsigned char* prow = smem + stage * Tr::kStageBytes + tl * 128;
#pragma unroll
        for (int c = 0; c < NH / 8; ++c) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * c + 2 * i;
            const float p0 = ex2_fast(x[r]);  // 2^-inf = 0
            const float p1 = ex2_fast(x[r + 1]);
            add_x2(lpart[r], lpart[r + 1], p0, p1);
            split_pair<T>(p0, p1, hi[i], lo[i]);
          }
          const int col = r0 + 8 * c;
          *reinterpret_cast<uint4*>(prow + (col / 64) * Tr::kSlab + ((((col % 64) >> 3) ^ (tl & 7)) << 4)) =
              make_uint4(hi[0], hi[1], hi[2], hi[3]);
          const int lcol = Tr::kPW / 2 + col;
          *reinterpret_cast<uint4*>(prow + (lcol / 64) * Tr::kSlab + ((((lcol % 64) >> 3) ^ (tl & 7)) << 4)) =
              make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // V rows past the tile's valid tokens may hold anything (NaN in unwritten
      // slots, stale rows of earlier tiles): zero those that the P V product
      // reads (up to the 16-token step holding the last valid token; an empty
      // tile's one step) so that 0 * V stays 0
      const int v_end = max(16, (n_valid + 15) / 16 * 16);
      if (n_valid < v_end) {
        unsigned char* vt = smem + stage * Tr::kStageBytes + 2 * Tr::kSlab;
        const int per_slab = (v_end - n_valid) * 8;
        for (int i = sg * 128 + tl; i < 2 * per_slab; i += 256) {
          const int hf = i / per_slab;
          const int rem = i - hf * per_slab;
          *reinterpret_cast<uint4*>(vt + hf * Tr::kSlab + (n_valid + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();  // P^T and the zeroed rows are read by the tensor cores
      // Observe every P V completion in order (the product of tile j - 1 was
      // issued right after S of this tile, so this rarely waits): pv_done then
      // never runs more than one phase ahead of this warp's parity waits.
      if (j >= 1 && !wait_pv(j - 1)) {
        failed = true;
        break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);

      if (flags & kTileLast) {
        // epilogue: tmp = the group's row sums of weights (final once this tile's P
        // is written, so reduced while its P V product runs), inv = their
        // reciprocals; then O is complete once P V of this tile is
        if (!group_reduce<NH, false>(lpart, red, tmp, my_grp, gk, q4, lane, abort_flag)) {
          failed = true;
          break;
        }
        if (lane < NH) inv[lane] = tmp[lane] > 0.f ? 1.f / tmp[lane] : 0.f;
        __syncwarp();
        if (!wait_pv(j)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const int us = hd.x, ukv = hd.y & 0xffff, up = hd.z & 0xffff, un = hd.z >> 16;
        const int rows = min(Tq, Lq - rt * Tq) * G;  // real rows of this tile
        const size_t row0 = (size_t)us * Lq + (size_t)rt * Tq;  // (sequence, first query token)
        if (un != 1 || NH > kKtMaxBulkRuns * G) {
          // short runs: thread tl stores dimension tl of each row (a warp's store
          // is 32 consecutive floats); the stage holds no output rows
          if (warp == 2 + 4 * sg && lane == 0) mbar_arrive(&empty[stage]);
          int tq = r0 / G, g = r0 - (r0 / G) * G;  // query token and head of row r0 + r
#pragma unroll
          for (int c = 0; c < NH / 8; ++c) {
            uint32_t vh[8], vl[8];
            tmem_ld8(tlane + Tr::kOCol + (uint32_t)(r0 + 8 * c), vh);
            tmem_ld8(tlane + Tr::kOCol + (uint32_t)(Tr::kPW / 2 + r0 + 8 * c), vl);
            tmem_wait_ld();
            tmem_pin8(vh);
            tmem_pin8(vl);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 8 * c + i;
              if (r0 + r < rows) {
                const size_t sh = (row0 + tq) * prm.num_heads + (size_t)ukv * G + g;
                const float v = __uint_as_float(vh[i]) + __uint_as_float(vl[i]);
                if (un == 1)
                  prm.out[sh * D + tl] = v * inv[r];
                else
                  prm.ws_acc[(sh * prm.max_parts + up) * D + tl] = v;
              }
              if (++g == G) {
                g = 0;
                ++tq;
              }
            }
          }
          if (un != 1 && tl < NH && r0 + tl < rows) {
            const int R = r0 + tl;
            const size_t sh = (row0 + R / G) * prm.num_heads + (size_t)ukv * G + R % G;
            prm.ws_ml[sh * prm.max_parts + up] = make_float2(mref[tl], tmp[tl]);
          }
          tc_fence_before();
          continue;
        }
        // Long runs (final rows): the group's rows go through the tile's V slabs
        // (dead once P V is complete; the stage stays held until the rows are
        // stored): thread tl writes dimension tl of each row, then one thread
        // stores each run of rows with the copy engine.
        float* stg = reinterpret_cast<float*>(smem + stage * Tr::kStageBytes + 2 * Tr::kSlab) + sg * NH * D;
#pragma unroll
        for (int c = 0; c < NH / 8; ++c) {
          uint32_t vh[8], vl[8];
          tmem_ld8(tlane + Tr::kOCol + (uint32_t)(r0 + 8 * c), vh);
          tmem_ld8(tlane + Tr::kOCol + (uint32_t)(Tr::kPW / 2 + r0 + 8 * c), vl);
          tmem_wait_ld();
          tmem_pin8(vh);
          tmem_pin8(vl);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 8 * c + i;  // row r0 + r
            stg[r * D + tl] = (__uint_as_float(vh[i]) + __uint_as_float(vl[i])) * inv[r];
          }
        }
        fence_proxy_async_smem();  // the staged rows are read by the copy engine
        tc_fence_before();
        if (!group_sync(my_grp, gk, lane, abort_flag)) {
          failed = true;
          break;
        }
        if (warp == 2 + 4 * sg && lane == 0) {
          // runs of rows of one query token are consecutive query heads
          const int r_end = min(r0 + NH, rows);
          for (int R = r0; R < r_end;) {
            const int tq = R / G, g = R - tq * G;
            const int run = min(r_end - R, G - g);
            bulk_store(prm.out + ((row0 + tq) * prm.num_heads + (size_t)ukv * G + g) * D, stg + (R - r0) * D,
                       (uint32_t)(run * D * 4));
            R += run;
          }
          bulk_commit();
          bulk_wait_read();
          mbar_arrive(&empty[stage]);
        }
      }
    }
    bulk_wait_all();  // this thread's output stores are complete
    if (failed && lane == 0) {
      flag_error(PKV_DEV_WAIT_TIMEOUT);
      *abort_flag = 1;
    }
  }

  // free the tensor memory once every role is done with it
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Tr::kTmemCols)
                 : "memory");
  }
}

}  // namespace pkv
