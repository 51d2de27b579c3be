// Paged attention for many query rows per K/V head on the 5th-generation tensor
// cores (tcgen05, sm_100a): the verify pass of speculative decoding and chunked
// prefill, where Lq new tokens of a sequence (times G query heads per K/V head)
// attend its paged context ("vLLM PagedAttention and continuous batching",
// section 5 on chunked prefill; the multi-token generalisation of the decode in
// "PagedAttention - Efficient Memory Management for LLM Serving with vLLM",
// section "Method (PagedAttention + vLLM)").
//
// A unit is (sequence s, K/V head kvh, row tile rt, partition p) from the plan
// kernel's list.  Its R <= 128 query rows (row r = query token rt*Tq + r/G, query
// head kvh*G + r%G) form the M = 128 operand of every MMA; the K/V context streams
// through 64-token tiles:
//
//   S = Q K^T           tcgen05.mma  M=128 N=64  K=D   (Q and the K tile from shared memory)
//   P = 2^(S*scale - m) four softmax warps, one row per thread, S read from tensor memory
//   O += P V            tcgen05.mma  M=128 N=D   K=64  (P from tensor memory, V as an MN-major operand)
//
// S (double-buffered, 2 x 64 columns), O (D columns) and P (double-buffered, 2 x
// 64 columns of packed 16-bit pairs) live in tensor memory: the softmax threads
// store P with tcgen05.st into their own lanes and the P V product reads it as its
// A operand, so P never touches shared memory, and the softmax of tile j+1
// overlaps the P V product of tile j.
// P is split into a 16-bit high part and the 16-bit rounding of the rest, and both
// are multiplied (with P rounded to 16 bits alone the error exceeds 2e-3).  O is
// rescaled only when a row's running maximum grows by more than 2^8 (the partial
// sums stay exact in fp32; the final division uses the same reference maximum).
//
// Warp roles (one CTA per SM, persistent over the unit list):
//   warp 0     producer: the unit's query tile (one 4-D TMA box per 64 columns) and
//              the K half of each tile (2-D TMA boxes per (block, K/V head) run,
//              128-byte swizzle); it publishes each tile's header and run rows;
//   warp 7     V producer: the V half of each published tile, on the same barrier;
//   warp 1     allocates / frees the tensor memory; its lane 0 issues the S products;
//   warp 6     its lane 0 issues the P V products, in tile order, as each P is written
//              (the two issuers commit to their own barriers, so neither waits behind
//              the other's issue);
//   warps 2-5  softmax and epilogue; warp w reads tensor-memory lanes 32*(w%4) ...
//
// Every mbarrier wait is bounded (kWaitLimitCycles) and checks the CTA abort flag;
// before the tensor memory is freed the MMA thread waits for all its MMAs.
#pragma once

#include "decode_gqa.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // M: query rows per tile = tensor-memory lanes
constexpr int kTcTile = 64;           // tokens per K/V tile
constexpr int kTcStages = 6;  // the P V product of tile t is issued after S of tile t + 2
constexpr int kTcThreads = 8 * 32;    // producer, S issuer, four softmax warps, P V issuer, V producer
constexpr int kTcPvWarp = 6;
constexpr int kTcVWarp = 7;
constexpr int kTcCtasPerSm = 1;       // shared memory (and tensor memory) per CTA
constexpr int kTcTmemCols = 512;      // S[2] at columns 0 and 64, O at 128, P[2] (high, low) at 256 and 320
constexpr float kTcRescaleLog2 = 8.0f;

struct TcParams {
  CUtensorMap tmap_k;  // 2-D view [NB*Hkv*B rows][D] of the K pool, box {64, unit_rows}, 128B swizzle
  CUtensorMap tmap_v;
  CUtensorMap tmap_q;  // 4-D view [S][Lq][Hq][D] of q, box {64, G, Tq, 1}, 128B swizzle
  const int32_t* block_tables;
  int num_heads;       // Hq
  int num_kv_heads;    // Hkv
  int group;           // G
  int q_len;           // Lq
  int tq_per_tile;     // Tq = floor(128 / G) query tokens per row tile
  int row_tiles;       // ceil(Lq / Tq)
  int block_size;
  int max_blocks;
  int num_blocks;
  float scale_log2;
  int part_tokens;
  int max_parts;
  float* out;          // [S][Lq][Hq][D]
  float* ws_acc;
  float2* ws_ml;
  const uint2* units;
  int* counters;
};

template <int D>
struct TcTraits {
  static constexpr int kHalves = D / 64;
  static constexpr int kSlabBytes = kTcTile * 128;          // 64 tokens x 64 columns
  static constexpr int kTileBytes = kHalves * kSlabBytes;   // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQSlabBytes = kTcRows * 128;         // 128 rows x 64 columns
  static constexpr int kQOffset = kTcStages * kStageBytes;
  static constexpr int kHdrOffset = kQOffset + kHalves * kQSlabBytes;  // two int4 per stage
  static constexpr int kRowsOffset = kHdrOffset + kTcStages * 32;  // [NS][32] pool rows of a tile's runs (-1: none)
  static constexpr int kBarOffset = kRowsOffset + kTcStages * 128;
  // full[NS], empty[NS], q_full, q_empty, s_full[2], s_free[2], p_full[2], o_done[2], drain[2], meta[NS]
  static constexpr int kNumBars = 3 * kTcStages + 12;
  static constexpr int kTmemSlotOffset = kBarOffset + kNumBars * 8;
  static constexpr int kAbortOffset = kTmemSlotOffset + 8;
  static constexpr int kSmemBytes = kAbortOffset + 8;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;      // the base is rounded up to 1024 bytes
  static constexpr uint32_t kOCol = 128;
  static constexpr uint32_t kPCol = 256;  // P buffer b: high part at kPCol + 64 b, low part 32 columns on
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(kQOffset % 1024 == 0, "swizzle atoms are 1024-byte aligned");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA");
};

// ---- tcgen05 helpers ---------------------------------------------------------

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start, leading
// and stride byte offsets in 16-byte units, version 1, layout type 2).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Operand format code of kind::f16 (fp16 = 0, bf16 = 1).
template <typename T>
struct TcFormat;
template <>
struct TcFormat<__half> {
  static constexpr uint32_t kCode = 0;
};
template <>
struct TcFormat<__nv_bfloat16> {
  static constexpr uint32_t kCode = 1;
};

// Instruction descriptor for kind::f16 with fp32 accumulation: A and B of one type
// (both fp16 or both bf16), A K-major, B K-major or MN-major, M x N.
template <typename T>
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (TcFormat<T>::kCode << 7) | (TcFormat<T>::kCode << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with the A operand (K-major, 16-bit pairs per 32-bit column) in tensor memory.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Redefine 32 registers after a tcgen05.wait::ld so that no use is scheduled above it.
__device__ __forceinline__ void tmem_pin32(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Wait for this thread's tensor-memory loads, then pin the loaded registers after
// the wait (the empty asm redefines them, so no use is scheduled above it).
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// (p0, p1) -> high parts (p in T) and low parts (T rounding of p - high), each as a
// packed pair; high + low carries ~16 more bits of p than high alone.
template <typename T>
__device__ __forceinline__ void split_pair(float p0, float p1, uint32_t& hi, uint32_t& lo);
template <>
__device__ __forceinline__ void split_pair<__nv_bfloat16>(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  hi = Mma16816<__nv_bfloat16>::pack(p0, p1);
  // a bf16 is the top half of an fp32
  lo = Mma16816<__nv_bfloat16>::pack(p0 - __uint_as_float(hi << 16), p1 - __uint_as_float(hi & 0xffff0000u));
}
template <>
__device__ __forceinline__ void split_pair<__half>(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  hi = Mma16816<__half>::pack(p0, p1);
  __half2 h;
  memcpy(&h, &hi, 4);
  const float2 f = __half22float2(h);
  lo = Mma16816<__half>::pack(p0 - f.x, p1 - f.y);
}

// (d0, d1) += (a0, a1): two fp32 additions in one packed instruction (sm_100), each
// rounded as a scalar addition.
__device__ __forceinline__ void add_x2(float& d0, float& d1, float a0, float a1) {
  uint64_t d, a;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
  asm("add.rn.f32x2 %0, %0, %1;" : "+l"(d) : "l"(a));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

// (d0, d1) *= (a0, a1): two fp32 multiplications in one packed instruction (sm_100).
__device__ __forceinline__ void mul_x2(float& d0, float& d1, float a0, float a1) {
  uint64_t d, a;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(d) : "l"(a));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

struct TcUnit {
  int s, kvh, rt, p, t_begin, t_end, n_parts, ctx;
};

// grid = min(#SMs, units); block = kTcThreads; one CTA per SM (shared memory).
template <typename T, int D>
__global__ void __launch_bounds__(kTcThreads, 1) paged_multi_query_tc_kernel(const __grid_constant__ TcParams prm) {
  using Tr = TcTraits<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* full = bars;
  uint64_t* empty = bars + kTcStages;
  uint64_t* q_full = bars + 2 * kTcStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_full + 2;  // [2]
  uint64_t* s_free = q_full + 4;  // [2]
  uint64_t* p_full = q_full + 6;  // [2]: P buffer b of tile j = j & 1 written
  uint64_t* o_done = q_full + 8;  // [2]: P V of tile j (j & 1 = b) complete
  uint64_t* drain = q_full + 10;  // [2]: one per MMA issuer
  uint64_t* meta = q_full + 12;   // [NS]: a tile's header and run rows are published
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
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&meta[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&s_free[0], 4);
    mbar_init(&s_free[1], 4);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // query rows that no TMA box covers (rows >= G * Tq) must read as zero
  for (int i = threadIdx.x; i < Tr::kHalves * Tr::kQSlabBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + Tr::kQOffset)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTcTmemCols)
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
    const int unit_rows = min(B, kTcTile);
    const int units_per_tile = kTcTile / unit_rows;
    const uint32_t run_bytes = (uint32_t)(unit_rows * 128);
    const uint32_t q_bytes = (uint32_t)(Tr::kHalves * 128 * G * Tq);

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

    int u = (int)blockIdx.x;
    TcUnit cur = describe(u, entry(u));
    int it = 0;  // tiles issued
    int nu = 0;  // query tiles issued
    bool stop = false;
    while (!stop) {
      const bool done = (long long)u >= total_units;
      const int u_next_lane0 = done ? 0 : claim();
      int u_next = 0;
      uint2 e_next = make_uint2(0u, 0u);
      if (!done) {
        // the previous unit's S products must be done reading the query tile
        int ok = 1;
        if (nu > 0 && lane == 0) ok = mbar_wait_bounded(q_empty, (nu - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) {
            flag_error(PKV_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, q_bytes);
#pragma unroll
          for (int hf = 0; hf < Tr::kHalves; ++hf)
            tma_load_4d(smem + Tr::kQOffset + hf * Tr::kQSlabBytes, &prm.tmap_q, hf * 64, cur.kvh * G,
                        cur.rt * Tq, cur.s, q_full, policy);
        }
        ++nu;
      }
      const int n_tok = max(0, cur.t_end - cur.t_begin);
      const int n_tiles = done ? 1 : max(1, (n_tok + kTcTile - 1) / kTcTile);
      const int32_t* table = prm.block_tables + (size_t)cur.s * prm.max_blocks;

      for (int i = 0; i < n_tiles; ++i, ++it) {
        const int stage = it % kTcStages;
        const int tile_t0 = cur.t_begin + i * kTcTile;
        const int u_t0 = tile_t0 + lane * unit_rows;
        const bool mine = !done && lane < units_per_tile && u_t0 < cur.t_end;
        const int phys = mine ? __ldg(table + u_t0 / B) : -1;  // u_t0 < ctx <= max_blocks * B
        if (it >= kTcStages) {
          int ok = 1;
          if (lane == 0) ok = mbar_wait_bounded(&empty[stage], ((it / kTcStages) - 1) & 1, abort_flag);
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
        const int n_valid = done ? 0 : max(0, min(kTcTile, cur.t_end - tile_t0));
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
          mbar_arrive_expect_tx(&full[stage], (uint32_t)__popc(loads) * 2u * Tr::kHalves * run_bytes);
          mbar_arrive(&meta[stage]);
        }
        if (load) {
          unsigned char* kt = smem + stage * Tr::kStageBytes + lane * unit_rows * 128;
#pragma unroll
          for (int hf = 0; hf < Tr::kHalves; ++hf)
            tma_load_2d(kt + hf * Tr::kSlabBytes, &prm.tmap_k, hf * 64, y, &full[stage], policy);
        }
        if (i == 0 && !done) {
          u_next = __shfl_sync(0xffffffffu, u_next_lane0, 0);
          e_next = entry(u_next);
        }
      }
      if (done || stop) break;
      u = u_next;
      cur = describe(u, e_next);
    }
    pdl_launch_dependents();
    // never leave with copies in flight into this CTA's shared memory
    if (lane == 0) {
      int no_abort = 0;
      for (int j = max(0, it - kTcStages); j < it; ++j)
        if (!mbar_wait_bounded(&full[j % kTcStages], (j / kTcStages) & 1, &no_abort))
          flag_error(PKV_DEV_WAIT_TIMEOUT);
      if (nu > 0 && !mbar_wait_bounded(q_full, (nu - 1) & 1, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
  } else if (warp == kTcVWarp) {
    // ------------------------------ V producer ------------------------------
    // Follows the producer tile by tile: once a tile is published (meta), each run's V
    // rows go to the stage's V half, completing on the same barrier.
    const uint64_t policy = l2_evict_first();
    const int unit_rows = min(prm.block_size, kTcTile);
    for (int t = 0;; ++t) {
      const int stage = t % kTcStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&meta[stage], (t / kTcStages) & 1, abort_flag))) {
        if (lane == 0) {
          flag_error(PKV_DEV_WAIT_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      if ((hdr[2 * stage].w >> 16) & kTileEnd) break;
      const int y = run_rows[stage * 32 + lane];
      if (y >= 0) {
        unsigned char* vt = smem + stage * Tr::kStageBytes + Tr::kTileBytes + lane * unit_rows * 128;
#pragma unroll
        for (int hf = 0; hf < Tr::kHalves; ++hf)
          tma_load_2d(vt + hf * Tr::kSlabBytes, &prm.tmap_v, hf * 64, y, &full[stage], policy);
      }
    }
  } else if (warp == 1 || warp == kTcPvWarp) {
    // ----------------------------- MMA issuers -----------------------------
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc<T>(kTcRows, kTcTile, false);
      constexpr uint32_t kIdescO = umma_idesc<T>(kTcRows, D, true);
      const uint32_t q_base = smem_addr(smem + Tr::kQOffset);
      bool ok = true;
      if (warp == 1) {
        // S of tile t as soon as its K/V, the unit's query tile and its S buffer are ready
        int nu = 0;
        for (int it = 0;; ++it) {
          const int stage = it % kTcStages;
          if (!mbar_wait_bounded(&full[stage], (it / kTcStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int flags = hdr[2 * stage].w >> 16;
          if (flags & kTileEnd) break;
          if (flags & kTileFirst) {
            if (!mbar_wait_bounded(q_full, nu & 1, abort_flag)) {
              ok = false;
              break;
            }
            ++nu;
          }
          const int sb = it & 1;
          if (it >= 2 && !mbar_wait_bounded(&s_free[sb], ((it >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_base = smem_addr(smem + stage * Tr::kStageBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (uint32_t)(k & 3) * 32u;  // 16 columns = 32 bytes inside a slab
            const uint64_t a = umma_desc_sw128(q_base + (k >> 2) * Tr::kQSlabBytes + off, 16, 1024);
            const uint64_t b = umma_desc_sw128(k_base + (k >> 2) * Tr::kSlabBytes + off, 16, 1024);
            umma_f16(tmem_base + (uint32_t)(sb * kTcTile), a, b, kIdescS, k > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          if (flags & kTileLast) umma_commit(q_empty);
        }
      } else {
        // O += P V of tile t once its P is written; a unit's first tile starts O over
        // (the softmax writes that P only after the previous unit's rows are read)
        for (int it = 0;; ++it) {
          const int stage = it % kTcStages;
          // the stage is released by this thread's commit below, so its header stays valid
          if (!mbar_wait_bounded(&full[stage], (it / kTcStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int flags = hdr[2 * stage].w >> 16;
          if (flags & kTileEnd) break;
          const int pb = it & 1;
          if (!mbar_wait_bounded(&p_full[pb], (it >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool first = flags & kTileFirst;
          const uint32_t p_hi = tmem_base + Tr::kPCol + (uint32_t)(pb * 64);
          const uint32_t p_lo = p_hi + 32;
          const uint32_t v_base = smem_addr(smem + stage * Tr::kStageBytes + Tr::kTileBytes);
#pragma unroll
          for (int k = 0; k < kTcTile / 16; ++k) {  // 16 tokens = 8 columns of packed pairs
            const uint64_t b = umma_desc_sw128(v_base + k * 16 * 128, Tr::kSlabBytes, 1024);
            umma_f16_tmem_a(tmem_base + Tr::kOCol, p_hi + 8 * k, b, kIdescO, (first && k == 0) ? 0u : 1u);
            umma_f16_tmem_a(tmem_base + Tr::kOCol, p_lo + 8 * k, b, kIdescO, 1u);
          }
          umma_commit(&empty[stage]);
          umma_commit(&o_done[pb]);
        }
      }
      if (!ok) {
        flag_error(PKV_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA this thread issued must be complete before the tensor memory is freed
      uint64_t* my_drain = warp == 1 ? &drain[0] : &drain[1];
      umma_commit(my_drain);
      int no_abort = 0;
      if (!mbar_wait_bounded(my_drain, 0, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // --------------------------- softmax / epilogue ---------------------------
    const int q4 = warp & 3;          // tensor-memory lane quarter of this warp
    const int r = q4 * 32 + lane;     // query row of this thread
    const uint32_t trow = tmem_base + ((uint32_t)(q4 * 32) << 16);
    const int tq_local = r / G;
    const bool row_in_tile = r < G * Tq;
    float m_ref = -INFINITY, l = 0.f;
    int4 uh = make_int4(0, 0, 0, 0);  // header of the unit being accumulated
    bool have_unit = false;
    bool failed = false;
    // P V products confirmed complete, per P buffer (each o_done phase is waited in order)
    int pv_seen0 = 0, pv_seen1 = 0;
    auto wait_pv = [&](int t) {  // P V of tile t (t >= 0) complete
      const int b = t & 1, k = t >> 1;
      int& seen = b ? pv_seen1 : pv_seen0;
      if (k < seen) return true;
      if (!mbar_wait_bounded(&o_done[b], k & 1, abort_flag)) return false;
      seen = k + 1;
      return true;
    };

    // write this row of the finished unit: the final row, or the partition's state
    auto finalize = [&]() {
      const int us = uh.x, ukv = uh.y & 0xffff, urt = uh.y >> 16, up = uh.z & 0xffff, un = uh.z >> 16;
      const int tq = urt * Tq + tq_local;
      const bool real = row_in_tile && tq < prm.q_len;
      const size_t sh = ((size_t)us * prm.q_len + tq) * prm.num_heads + (size_t)ukv * G + (r - tq_local * G);
      const float f = un == 1 ? ((l > 0.f) ? 1.f / l : 0.f) : 1.f;
      float* dst_row = un == 1 ? prm.out + sh * D : prm.ws_acc + (sh * prm.max_parts + up) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + Tr::kOCol + 32 * c, v);
        tmem_wait_ld();
        tmem_pin32(v);
        if (real) {
          float4* dst = reinterpret_cast<float4*>(dst_row + 32 * c);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(v[4 * k]) * f, __uint_as_float(v[4 * k + 1]) * f,
                                 __uint_as_float(v[4 * k + 2]) * f, __uint_as_float(v[4 * k + 3]) * f);
        }
      }
      if (real && un != 1) prm.ws_ml[sh * prm.max_parts + up] = make_float2(m_ref, l);
    };

    for (int j = 0;; ++j) {
      const int stage = j % kTcStages;
      if (!mbar_wait_bounded(&full[stage], (j / kTcStages) & 1, abort_flag)) {
        failed = true;
        break;
      }
      const int4 hd = hdr[2 * stage];
      const int4 hd2 = hdr[2 * stage + 1];
      const int flags = hd.w >> 16;
      const int n_valid = hd.w & 0xffff;
      if (flags & kTileEnd) {
        // the last unit's products must be complete before its rows are read
        if ((j >= 2 && !wait_pv(j - 2)) || (j >= 1 && !wait_pv(j - 1))) {
          failed = true;
          break;
        }
        tc_fence_after();
        if (have_unit) finalize();
        break;
      }
      const int sb = j & 1;
      if (!mbar_wait_bounded(&s_full[sb], (j >> 1) & 1, abort_flag)) {
        failed = true;
        break;
      }
      tc_fence_after();
      float x[kTcTile];
      {
        uint32_t v[kTcTile];
        tmem_ld32(trow + (uint32_t)(sb * kTcTile), v);
        tmem_ld32(trow + (uint32_t)(sb * kTcTile + 32), v + 32);
        tmem_wait_ld();
        tmem_pin32(v);
        tmem_pin32(v + 32);
#pragma unroll
        for (int c = 0; c < kTcTile; ++c) x[c] = __uint_as_float(v[c]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      // causal limit of this row: query token tq sees positions < ctx - Lq + tq + 1
      const int t0 = hd2.x, ctx = hd2.y;
      const int tq = (hd.y >> 16) * Tq + tq_local;
      const int limit = (row_in_tile && tq < prm.q_len) ? ctx - prm.q_len + tq + 1 : 0;
      const int n_ok = max(0, min(n_valid, limit - t0));  // columns [0, n_ok) are visible
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTcTile; c += 2) {
        float s0 = x[c], s1 = x[c + 1];
        mul_x2(s0, s1, prm.scale_log2, prm.scale_log2);  // two columns per packed multiply
        x[c] = c < n_ok ? s0 : -INFINITY;
        x[c + 1] = c + 1 < n_ok ? s1 : -INFINITY;
        mt = fmaxf(mt, x[c]);
        mt = fmaxf(mt, x[c + 1]);
      }

      // P buffer j & 1 was last read by the P V product of tile j - 2
      if (j >= 2 && !wait_pv(j - 2)) {
        failed = true;
        break;
      }
      const bool first = flags & kTileFirst;
      const bool need = !first && mt > m_ref + kTcRescaleLog2;
      // O is touched (read for the previous unit's rows, or rescaled): every product so far must be done
      if ((first && have_unit) || __any_sync(0xffffffffu, need)) {
        if (j >= 1 && !wait_pv(j - 1)) {
          failed = true;
          break;
        }
        tc_fence_after();
        if (first) {
          finalize();
        } else {
          const float alpha = need ? ex2_fast(m_ref - mt) : 1.f;  // 0 while m_ref is -inf
          if (need) {
            l *= alpha;
            m_ref = mt;
          }
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t v[16];
            tmem_ld16(trow + Tr::kOCol + 16 * c, v);
            tmem_wait_ld16(v);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st16(trow + Tr::kOCol + 16 * c, v);
          }
          tmem_wait_st();
        }
      }
      if (first) {
        uh = hd;
        have_unit = true;
        m_ref = mt;
        l = 0.f;
      }

      // P = 2^(x - m_ref) as high + low 16-bit parts, written to this row's tensor-memory
      // lane: packed pairs, tokens 2c and 2c + 1 in column c
      uint32_t hi[kTcTile / 2], lo[kTcTile / 2];
      float l0 = 0.f, l1 = 0.f;  // row-sum partials of the even and odd tokens
#pragma unroll
      for (int c2 = 0; c2 < kTcTile / 2; ++c2) {
        const int c = 2 * c2;
        float t0 = x[c], t1 = x[c + 1];
        add_x2(t0, t1, -m_ref, -m_ref);  // x - m_ref, two tokens per packed add
        const float p0 = x[c] == -INFINITY ? 0.f : ex2_fast(t0);
        const float p1 = x[c + 1] == -INFINITY ? 0.f : ex2_fast(t1);
        add_x2(l0, l1, p0, p1);
        split_pair<T>(p0, p1, hi[c2], lo[c2]);
      }
      l += l0 + l1;
      {
        const uint32_t pcol = trow + Tr::kPCol + (uint32_t)(sb * 64);
        tmem_st16(pcol, *reinterpret_cast<uint32_t(*)[16]>(hi));
        tmem_st16(pcol + 16, *reinterpret_cast<uint32_t(*)[16]>(hi + 16));
        tmem_st16(pcol + 32, *reinterpret_cast<uint32_t(*)[16]>(lo));
        tmem_st16(pcol + 48, *reinterpret_cast<uint32_t(*)[16]>(lo + 16));
        tmem_wait_st();
      }
      // V rows past the tile's valid tokens may hold anything (NaN in unwritten
      // slots): zero them so that 0 * V stays 0
      if (n_valid < kTcTile) {
        unsigned char* vt = smem + stage * Tr::kStageBytes + Tr::kTileBytes;
        const int chunks = (kTcTile - n_valid) * 8 * Tr::kHalves;
        for (int i = (warp - 2) * 32 + lane; i < chunks; i += 128) {
          const int hf = i / ((kTcTile - n_valid) * 8);
          const int rem = i - hf * (kTcTile - n_valid) * 8;
          *reinterpret_cast<uint4*>(vt + hf * Tr::kSlabBytes + (n_valid + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      if (n_valid < kTcTile) fence_proxy_async_smem();  // the zeroed rows are read by the tensor cores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTcTmemCols)
                 : "memory");
  }
}

}  // namespace pkv
