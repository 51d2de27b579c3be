// Grouped-query paged decode on tensor cores (sm_100a), 16-bit K/V.
//
// With G = Hq / Hkv query heads per K/V head, one K/V tile serves G query rows,
// so the tile's work is a small dense contraction: S = Q K^T (G x tokens) and
// O += P V (G x D).  CUDA-core FMAs would cost ~2 G D per token and head, which
// at G = 8 outruns the HBM rate; the warp-level m16n8k16 MMA covers 16 query
// rows at once (G <= 16, padded), so the kernel stays bound by HBM.  (The
// tcgen05 MMA needs M >= 64 rows: at <= 16 real rows it would spend most of its
// work and tensor-memory traffic on padding.)
//
// Structure (persistent, one producer warp + 4 consumer warps, like the
// multi-head kernel in decode.cuh):
//  * unit = (sequence s, K/V head kvh, partition p); the plan kernel's list is
//    reused; CTA b starts with unit b, then takes units with an atomic counter.
//  * producer: for every run of rows of one (block, K/V head) in the tile, two
//    tensor-map TMA loads per 64 columns (K and V) into a 128-byte-swizzled
//    stage; the G query rows are one bulk copy at a unit's first tile.
//  * consumer warp w owns tokens [16w, 16w+16) of every 64-token tile:
//      S (16 rows x 16 tokens) = Q (16 x D) . K^T   -- ldmatrix + 2 MMAs per 16 dims
//      online softmax per row in base 2 (rows live in lane groups of 4)
//      O (16 x D) += P . V                          -- ldmatrix.trans + MMAs
//    P is split into hi + lo 16-bit parts and both are multiplied, so the
//    weights keep ~16 significant bits instead of 8 (bf16) or 11 (fp16).
//    Rows of V past the context are zeroed in shared memory before the MMA
//    (0 * NaN would poison the sum); logits past the context are set to -inf.
//  * at a unit's last tile the 4 warps' (m, l, O) states are merged through
//    shared memory and written as the output rows (or partition states for the
//    log-sum-exp merge kernel, shared with the multi-head path).
#pragma once

#include <cuda.h>

#include "decode.cuh"
#include "pkv_device.cuh"

namespace pkv {

constexpr int kGqaTile = 64;      // tokens per stage
constexpr int kGqaRows = 16;      // query rows of one MMA tile (G <= 16)

struct GqaParams {
  CUtensorMap tmap_k;  // 2-D view [NB*Hkv*B rows][D] of the K pool, box {64, unit_rows}, 128B swizzle
  CUtensorMap tmap_v;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int num_heads;     // Hq
  int num_kv_heads;  // Hkv
  int group;         // G = Hq / Hkv
  int q_len;         // Lq query tokens per sequence (1 = decode)
  int rows;          // Lq * G query rows per (sequence, K/V head); row r = (token r / G, head r % G)
  int row_tiles;     // ceil(rows / 16)
  int block_size;
  int max_blocks;
  int num_blocks;
  float scale_log2;
  int part_tokens;
  int max_parts;
  float* out;
  float* ws_acc;
  float2* ws_ml;
  const uint2* units;  // {(s << 16) | p, clamped context length} per live (sequence, partition)
  int* counters;
};

template <int D, int NS>
struct GqaTraits {
  static constexpr int kHalves = D / 64;                      // 64-column, 128-byte swizzled slabs
  static constexpr int kSlabBytes = kGqaTile * 128;           // one slab of a tile
  static constexpr int kTileBytes = kHalves * kSlabBytes;     // K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = kGqaRows * D * 2;            // query rows of a unit
  static constexpr int kQOffset = NS * kStageBytes;
  static constexpr int kHdrOffset = kQOffset + NS * kQBytes;   // NS x 2 int4 headers
  static constexpr int kBarOffset = kHdrOffset + NS * 32;
  static constexpr int kAbortOffset = kBarOffset + (2 * NS + 1) * 8;
  static constexpr int kRedMlOffset = (kAbortOffset + 16 + 127) / 128 * 128;
  static constexpr int kRedAccFloats = kConsumerWarps * kGqaRows * D;  // lives in the unit's last stage
  static constexpr int kRedMlFloats = kConsumerWarps * kGqaRows * 2;
  static constexpr int kSmemBytes = kRedMlOffset + kRedMlFloats * 4;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // the base is rounded up to 1024 bytes
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(kStageBytes % 1024 == 0, "swizzled slabs stay 1024-byte aligned");
  static_assert(kRedAccFloats * 4 <= kStageBytes, "the warps' row states fit in one stage");
};

// ---- PTX wrappers ------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <typename T>
struct Mma16816;

template <>
struct Mma16816<__nv_bfloat16> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  // two floats -> packed pair (round to nearest even); lo in the low half
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    uint32_t r;
    memcpy(&r, &v, 4);
    return r;
  }
  __device__ __forceinline__ static float2 unpack(uint32_t r) {
    __nv_bfloat162 v;
    memcpy(&v, &r, 4);
    return __bfloat1622float2(v);
  }
};

template <>
struct Mma16816<__half> {
  __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    uint32_t r;
    memcpy(&r, &v, 4);
    return r;
  }
  __device__ __forceinline__ static float2 unpack(uint32_t r) {
    __half2 v;
    memcpy(&v, &r, 4);
    return __half22float2(v);
  }
};

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled slab:
// the chunk index is XORed with the row index modulo 8 (the TMA 128B pattern on a
// 1024-byte-aligned slab).
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// A unit as the producer sees it: (sequence, K/V head, 16-row tile, partition).
struct GqaUnit {
  int s, kvh, rt, p, t_begin, t_end, n_parts, ctx;
};

// ---------------------------------------------------------------------------
// grid = min(#SMs x resident CTAs, units); block = kDecodeThreads (4 consumer warps + producer)
// ---------------------------------------------------------------------------
template <typename T, int D, int NS>
__global__ void __launch_bounds__(kDecodeThreads) paged_decode_gqa_kernel(const __grid_constant__ GqaParams prm) {
  using Tr = GqaTraits<D, NS>;
  using M = Mma16816<T>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::kBarOffset);
  uint64_t* empty = full + NS;
  uint64_t* epi = empty + NS;
  int4* hdr = reinterpret_cast<int4*>(smem + Tr::kHdrOffset);  // [stage][2]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Tr::kAbortOffset);
  float* red_ml = reinterpret_cast<float*>(smem + Tr::kRedMlOffset);  // [warp][row][2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Hq = prm.num_heads;
  const int Hkv = prm.num_kv_heads;
  const int G = prm.group;
  const int Lq = prm.q_len;
  const int RT = prm.row_tiles;
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
  // query slots: rows >= G are never written by a copy and must read as zero
  for (int i = threadIdx.x; i < NS * Tr::kQBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + Tr::kQOffset)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  __syncthreads();
  pdl_wait_primary();

  if (warp == kConsumerWarps) {
    // ------------------------------- producer -------------------------------
    const T* qg = static_cast<const T*>(prm.q);
    const uint64_t policy = l2_evict_first();
    const int B = prm.block_size;
    const int unit_rows = min(B, kGqaTile);
    const int units_per_tile = kGqaTile / unit_rows;
    const int per_sp = Hkv * RT;  // units per (sequence, partition)
    const long long total_units = (long long)prm.counters[1] * per_sp;
    const uint32_t row_bytes = (uint32_t)(D * 2);
    const uint32_t run_bytes = (uint32_t)(unit_rows * 128);  // one 64-column box

    auto describe = [&](int u, uint2 e) {
      GqaUnit d{0, 0, 0, 0, 0, 0, 1, 0};
      if ((long long)u < total_units) {
        d.s = (int)(e.x >> 16);
        d.p = (int)(e.x & 0xffffu);
        const int rem = u - (u / per_sp) * per_sp;
        d.kvh = rem / RT;
        d.rt = rem - d.kvh * RT;
        d.ctx = (int)e.y;  // clamped by the plan kernel
        d.t_begin = d.p * PT;
        d.t_end = min(d.ctx, d.t_begin + PT);
        d.n_parts = parts_of(d.ctx, PT);
      }
      return d;
    };
    // CTA b starts with unit b; later units come from the counter, offset by the grid
    // size (lane 0 claims; the caller broadcasts the id when it needs it)
    auto claim = [&]() { return lane == 0 ? (int)gridDim.x + atomicAdd(&prm.counters[0], 1) : 0; };
    auto entry = [&](int u) {
      return (long long)u < total_units ? __ldcg(prm.units + u / per_sp) : make_uint2(0u, 0u);
    };
    int u = (int)blockIdx.x;
    GqaUnit cur = describe(u, entry(u));
    int it = 0;  // stage iterations issued so far
    bool stop = false;
    while (!stop) {
      const bool done = (long long)u >= total_units;
      const int u_next_lane0 = done ? 0 : claim();  // one unit ahead
      int u_next = 0;
      uint2 e_next = make_uint2(0u, 0u);
      const int n_tok = max(0, cur.t_end - cur.t_begin);
      const int n_tiles = done ? 1 : max(1, (n_tok + kGqaTile - 1) / kGqaTile);
      const int32_t* table = prm.block_tables + (size_t)cur.s * prm.max_blocks;

      for (int i = 0; i < n_tiles; ++i, ++it) {
        const int stage = it % NS;
        const int tile_t0 = cur.t_begin + i * kGqaTile;
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
        const int n_valid = done ? 0 : max(0, min(kGqaTile, cur.t_end - tile_t0));
        bool load = false;
        if (mine) {
          if (phys >= 0 && phys < prm.num_blocks)
            load = true;
          else
            flag_error(PKV_DEV_BLOCK_ID);
        }
        const unsigned loads = __ballot_sync(0xffffffffu, load);
        const bool load_q = (i == 0) && n_tok > 0;
        const int nr = min(kGqaRows, prm.rows - cur.rt * kGqaRows);  // real query rows of this tile
        if (lane == 0) {
          const int flags = done ? kTileEnd : ((i == 0 ? kTileFirst : 0) | (i == n_tiles - 1 ? kTileLast : 0));
          hdr[2 * stage] = make_int4(cur.s, cur.kvh | (cur.rt << 16), cur.p | (cur.n_parts << 16),
                                     n_valid | (flags << 16));
          hdr[2 * stage + 1] = make_int4(tile_t0, cur.ctx, 0, 0);
          const uint32_t tx = (uint32_t)__popc(loads) * 2u * Tr::kHalves * run_bytes +
                              (load_q ? (uint32_t)nr * row_bytes : 0u);
          mbar_arrive_expect_tx(&full[stage], tx);
        }
        __syncwarp();
        if (load) {
          // rows of this (block, K/V head) run in the 2-D view: ((phys * Hkv + kvh) * B + offset)
          const int y = (phys * Hkv + cur.kvh) * B + (u_t0 % B);
          unsigned char* kt = smem + stage * Tr::kStageBytes + lane * unit_rows * 128;
#pragma unroll
          for (int hf = 0; hf < Tr::kHalves; ++hf) {
            tma_load_2d(kt + hf * Tr::kSlabBytes, &prm.tmap_k, hf * 64, y, &full[stage], policy);
            tma_load_2d(kt + Tr::kTileBytes + hf * Tr::kSlabBytes, &prm.tmap_v, hf * 64, y, &full[stage], policy);
          }
        }
        if (load_q && lane < nr) {  // query row r = (token r / G, head-in-group r % G)
          const int r = cur.rt * kGqaRows + lane;
          const int tq = r / G;
          const size_t src = (((size_t)cur.s * Lq + tq) * Hq + (size_t)cur.kvh * G + (r - tq * G)) * D;
          bulk_load(smem + Tr::kQOffset + stage * Tr::kQBytes + lane * row_bytes, qg + src, row_bytes, &full[stage],
                    policy);
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
    pdl_launch_dependents();
    if (lane == 0) {
      int no_abort = 0;
      for (int j = max(0, it - NS); j < it; ++j)
        if (!mbar_wait_bounded(&full[j % NS], (j / NS) & 1, &no_abort)) flag_error(PKV_DEV_WAIT_TIMEOUT);
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int gid = lane >> 2;  // row group: rows gid and gid + 8
  const int t4 = lane & 3;    // column pair within an 8-column MMA tile
  const int tok0 = warp * 16; // this warp's 16 tokens of every tile
  constexpr int KS = D / 16;  // 16-dimension steps
  constexpr int DT = D / 8;   // 8-dimension output tiles

  uint32_t qa[KS][4];
  float o[DT][4];
  float m_r[2], l_r[2];
  int units_done = 0;
#pragma unroll
  for (int j = 0; j < DT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  m_r[0] = m_r[1] = -INFINITY;
  l_r[0] = l_r[1] = 0.f;
#pragma unroll
  for (int j = 0; j < KS; ++j) qa[j][0] = qa[j][1] = qa[j][2] = qa[j][3] = 0u;

  // ldmatrix row addresses (relative to a slab) for this lane
  const int lm = lane >> 3;  // which 8x8 matrix of the x4 load this lane addresses
  const int lr = lane & 7;   // row within it

  for (int it = 0;; ++it) {
    const int stage = it % NS;
    if (!mbar_wait_bounded(&full[stage], (it / NS) & 1, abort_flag)) {
      if (lane == 0) {
        flag_error(PKV_DEV_WAIT_TIMEOUT);
        *abort_flag = 1;
      }
      break;
    }
    const int4 hd = hdr[2 * stage];
    const int4 hd2 = hdr[2 * stage + 1];
    const int flags = hd.w >> 16;
    const int n_valid = hd.w & 0xffff;
    if (flags & kTileEnd) break;
    unsigned char* kt = smem + stage * Tr::kStageBytes;
    unsigned char* vt = kt + Tr::kTileBytes;
    const int rt = hd.y >> 16;
    const int nr = min(kGqaRows, prm.rows - rt * kGqaRows);  // real rows of this unit's tile
    // causal limit of rows gid and gid + 8: query token tq sees positions < ctx - Lq + tq + 1
    int lim[2];
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const int rho = gid + 8 * hrow;
      const int tq = (rt * kGqaRows + rho) / G;
      lim[hrow] = rho < nr ? min(n_valid, hd2.y - Lq + tq + 1 - hd2.x) : 0;
    }

    if (flags & kTileFirst) {
#pragma unroll
      for (int j = 0; j < DT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      m_r[0] = m_r[1] = -INFINITY;
      l_r[0] = l_r[1] = 0.f;
      const uint32_t* qs = reinterpret_cast<const uint32_t*>(smem + Tr::kQOffset + stage * Tr::kQBytes);
#pragma unroll
      for (int j = 0; j < KS; ++j) {  // A fragment: rows gid / gid+8, dims 16j + 2 t4 (+8)
        qa[j][0] = qs[(gid * D + 16 * j + 2 * t4) / 2];
        qa[j][1] = qs[((gid + 8) * D + 16 * j + 2 * t4) / 2];
        qa[j][2] = qs[(gid * D + 16 * j + 8 + 2 * t4) / 2];
        qa[j][3] = qs[((gid + 8) * D + 16 * j + 8 + 2 * t4) / 2];
      }
    }

    // rows of V past the context: zero this warp's ones (they may hold NaN)
    const bool partial = n_valid < tok0 + 16;
    if (partial) {
      for (int r = max(n_valid, tok0) + (lane >> 3); r < tok0 + 16; r += 4) {
#pragma unroll
        for (int hf = 0; hf < Tr::kHalves; ++hf)
          *reinterpret_cast<uint4*>(vt + hf * Tr::kSlabBytes + r * 128 + (lane & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // ---- S = Q K^T for this warp's 16 tokens (two 8-token MMA tiles) ----
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
    if (n_valid > tok0) {
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        // matrices: (tokens 0-7, dims 16j..+7), (tokens 0-7, dims +8..), (tokens 8-15, ..), (tokens 8-15, +8..)
        const int row = tok0 + ((lm >> 1) << 3) + lr;
        const int chunk = 2 * j + (lm & 1);
        uint32_t b[4];
        ldsm_x4(smem_addr(kt + (chunk >> 3) * Tr::kSlabBytes + swz(row, chunk & 7)), b);
        M::run(sacc[0], qa[j], b[0], b[1]);
        M::run(sacc[1], qa[j], b[2], b[3]);
      }
    }

    // ---- online softmax (base 2) per row; columns a row may not see are -inf ----
    // Rows 8..15 (the second half of every fragment) are padding when nr <= 8.
    const int halves = nr > 8 ? 2 : 1;
    float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = tok0 + nt * 8 + 2 * t4 + (c & 1);
        const float v = (tok < lim[c >> 1] && (c >> 1) < halves) ? sacc[nt][c] * prm.scale_log2 : -INFINITY;
        sacc[nt][c] = v;
        mt[c >> 1] = fmaxf(mt[c >> 1], v);
      }
    float alpha[2] = {1.f, 1.f};
    float mnew[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      if (hrow >= halves) break;
      mt[hrow] = fmaxf(mt[hrow], __shfl_xor_sync(0xffffffffu, mt[hrow], 1));
      mt[hrow] = fmaxf(mt[hrow], __shfl_xor_sync(0xffffffffu, mt[hrow], 2));
      mnew[hrow] = fmaxf(m_r[hrow], mt[hrow]);
      alpha[hrow] = (mnew[hrow] == -INFINITY) ? 1.f : ex2_fast(m_r[hrow] - mnew[hrow]);  // 0 when m was -inf
      m_r[hrow] = mnew[hrow];
      l_r[hrow] *= alpha[hrow];
    }
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
      for (int j = 0; j < DT; ++j) {
        o[j][0] *= alpha[0];
        o[j][1] *= alpha[0];
        o[j][2] *= alpha[1];
        o[j][3] *= alpha[1];
      }
    }
    // P = 2^(s - m); split into hi + lo 16-bit parts for the PV products
    uint32_t pa_hi[4], pa_lo[4];
    {
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float mm = mnew[c >> 1];
          const float e = (mm == -INFINITY) ? 0.f : ex2_fast(sacc[nt][c] - mm);
          p[nt][c] = e;
          l_r[c >> 1] += e;
        }
      // A fragment of P (k = tokens): a0 = (row gid, tokens 2t4 of tile 0), a1 = (row gid+8, ...),
      // a2 = (row gid, tile 1), a3 = (row gid+8, tile 1)
      const float pv[4][2] = {{p[0][0], p[0][1]}, {p[0][2], p[0][3]}, {p[1][0], p[1][1]}, {p[1][2], p[1][3]}};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pa_hi[k] = M::pack(pv[k][0], pv[k][1]);
        const float2 h = M::unpack(pa_hi[k]);
        pa_lo[k] = M::pack(pv[k][0] - h.x, pv[k][1] - h.y);
      }
    }

    // ---- O += P V (16 tokens x D) ----
    if (n_valid > tok0) {
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        // matrices: (tokens 0-7, dims 16i..+7), (tokens 8-15, dims 16i..), (tokens 0-7, +8..), (tokens 8-15, +8..)
        const int row = tok0 + ((lm & 1) << 3) + lr;
        const int chunk = 2 * i + (lm >> 1);
        uint32_t b[4];
        ldsm_x4_trans(smem_addr(vt + (chunk >> 3) * Tr::kSlabBytes + swz(row, chunk & 7)), b);
        M::run(o[2 * i], pa_hi, b[0], b[1]);
        M::run(o[2 * i], pa_lo, b[0], b[1]);
        M::run(o[2 * i + 1], pa_hi, b[2], b[3]);
        M::run(o[2 * i + 1], pa_lo, b[2], b[3]);
      }
    }
    if (!(flags & kTileLast)) {
      if (partial) fence_proxy_async_smem();  // generic writes above, async (TMA) writes next
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      continue;
    }

    // ---- unit epilogue: the 4 warps hold disjoint tokens; merge their rows in
    //      the stage just consumed, then hand the stage back to the producer ----
    float lsum[2];
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      float v = l_r[hrow];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      lsum[hrow] = v;
    }
    // every warp has finished reading this stage's K and V before it is overwritten
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
    float* red_acc = reinterpret_cast<float*>(kt);  // [warp][row][D] over the consumed stage
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const int row = gid + 8 * hrow;
      if (row < nr) {
        float* dst = red_acc + (warp * kGqaRows + row) * D;
#pragma unroll
        for (int j = 0; j < DT; ++j) {
          dst[j * 8 + 2 * t4] = o[j][2 * hrow];
          dst[j * 8 + 2 * t4 + 1] = o[j][2 * hrow + 1];
        }
        if (t4 == 0) {
          red_ml[(warp * kGqaRows + row) * 2] = m_r[hrow];
          red_ml[(warp * kGqaRows + row) * 2 + 1] = lsum[hrow];
        }
      }
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
    const int us = hd.x, ukv = hd.y & 0xffff, up = hd.z & 0xffff, un = hd.z >> 16;
    for (int idx = threadIdx.x; idx < nr * D; idx += kConsumerWarps * 32) {
      const int row = idx / D;
      const int d = idx - row * D;
      const int r = rt * kGqaRows + row;
      const int tq = r / G;
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, red_ml[(w * kGqaRows + row) * 2]);
      float L = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = red_ml[(w * kGqaRows + row) * 2];
        const float sc = (mx == -INFINITY) ? 0.f : ex2_fast(mw - mx);
        L = fmaf(red_ml[(w * kGqaRows + row) * 2 + 1], sc, L);
        acc = fmaf(red_acc[(w * kGqaRows + row) * D + d], sc, acc);
      }
      const size_t sh = ((size_t)us * Lq + tq) * Hq + (size_t)ukv * G + (r - tq * G);
      if (un == 1) {
        prm.out[sh * D + d] = (L > 0.f) ? acc / L : 0.f;
      } else {
        const size_t ws = sh * prm.max_parts + up;
        prm.ws_acc[ws * D + d] = acc;
        if (d == 0) prm.ws_ml[ws] = make_float2(mx, L);
      }
    }
    // every consumer thread has read the states before the stage goes back to the
    // producer; the generic writes are ordered before the next TMA writes
    fence_proxy_async_smem();
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
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
}

}  // namespace pkv
