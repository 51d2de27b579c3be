// Paged single-query decode attention for sm_100a.
//
// Three kernels, launched back to back on one stream:
//
//  1. paged_decode_plan_kernel (1 CTA): turns context_lens into a compact list of
//     live (sequence, partition) work units and resets the unit counter.
//  2. paged_decode_kernel (persistent, one or more CTAs per SM): every CTA takes
//     units from the counter until none are left.  A unit is (sequence s, head h,
//     partition p).  The CTA streams the unit's K and V rows through a ring of
//     NS shared-memory stages:
//       producer warp  follows the block table and issues one bulk (TMA-engine)
//                      copy per contiguous (block, head) run of rows, plus the q
//                      row at a unit's first tile; it writes a small header per
//                      stage (unit, valid rows, first/last flags) and announces
//                      the stage's bytes on its "full" mbarrier.  It runs ahead
//                      across unit boundaries, so the ring never drains between
//                      units.
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
//  3. paged_decode_merge_kernel: log-sum-exp merge of the partitions of every
//     (sequence, head) whose context spans more than one partition.
//
// "Gather the non-contiguous blocks along the block table and compute
// softmax(QK^T)V" ("PagedAttention - Efficient Memory Management for LLM Serving
// with vLLM", section "Method (PagedAttention + vLLM)"): the gather is done by the
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

struct DecodeParams {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int num_heads;
  int block_size;
  int max_blocks;
  int num_blocks;
  float scale_log2;   // scale * log2(e): logits are kept in base 2
  int part_tokens;    // tokens per partition; >= max_blocks * block_size when not splitting
  int max_parts;      // partitions a context can span (workspace stride)
  float* out;         // [S][H][D]
  float* ws_acc;      // [S][H][max_parts][D]   (split only)
  float2* ws_ml;      // [S][H][max_parts]      (split only)
  const uint32_t* units;  // (s << 16) | p for each live (sequence, partition)
  int* counters;          // [0] unit counter, [1] number of live (sequence, partition)
};

__device__ __forceinline__ int clamp_ctx(int ctx, int max_ctx) { return ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx); }

// Number of partitions a context of ctx tokens occupies; an empty context still
// gets one unit so that its output row is written (as zeros).
__device__ __forceinline__ int parts_of(int ctx, int part_tokens) {
  const int n = (ctx + part_tokens - 1) / part_tokens;
  return n < 1 ? 1 : n;
}

// ---------------------------------------------------------------------------
// 1. plan: compact list of live (sequence, partition) units.  One CTA of 1024.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
    paged_decode_plan_kernel(const int32_t* __restrict__ context_lens, int num_seqs, int max_ctx, int part_tokens,
                             uint32_t* __restrict__ units, int* __restrict__ counters) {
  __shared__ int warp_sums[kPlanThreads / 32];
  const int tid = threadIdx.x;
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
  const int lane = tid & 31, warp = tid >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) {
      counters[0] = 0;
      counters[1] = wi;
    }
  }
  __syncthreads();
  int pos = warp_sums[warp] + incl - mine;
  for (int s = s0; s < s1; ++s) {
    const int n = parts_of(clamp_ctx(context_lens[s], max_ctx), part_tokens);
    for (int p = 0; p < n; ++p) units[pos++] = ((uint32_t)s << 16) | (uint32_t)p;
  }
}

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
  const int max_ctx = prm.max_blocks * prm.block_size;
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

    int u = 0;
    if (lane == 0) u = atomicAdd(&prm.counters[0], 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    int it = 0;  // stage iterations issued so far
    bool stop = false;
    while (!stop) {
      const bool done = (long long)u >= total_units;
      int s = 0, h = 0, p = 0, t_begin = 0, t_end = 0, n_parts = 1;
      if (!done) {
        const uint32_t sp = prm.units[u / H];
        s = (int)(sp >> 16);
        p = (int)(sp & 0xffffu);
        h = u - (u / H) * H;
        const int ctx = clamp_ctx(prm.context_lens[s], max_ctx);
        t_begin = p * PT;
        t_end = min(ctx, t_begin + PT);
        n_parts = parts_of(ctx, PT);
      }
      int u_next = 0;
      if (!done && lane == 0) u_next = atomicAdd(&prm.counters[0], 1);  // used after this unit
      const int n_tok = max(0, t_end - t_begin);
      const int n_tiles = done ? 1 : max(1, (n_tok + TT - 1) / TT);
      const int32_t* table = prm.block_tables + (size_t)s * prm.max_blocks;

      for (int i = 0; i < n_tiles; ++i, ++it) {
        const int stage = it % NS;
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
        const int tile_t0 = t_begin + i * TT;
        const int n_valid = done ? 0 : max(0, min(TT, t_end - tile_t0));
        uint32_t bytes = 0;
        size_t src_off = 0;
        if (lane < units_per_tile) {
          const int u_t0 = tile_t0 + lane * unit_rows;
          if (u_t0 < t_end) {
            const int rows = min(unit_rows, t_end - u_t0);
            const int phys = __ldg(table + u_t0 / B);  // u_t0 < ctx <= max_blocks * B
            if (phys >= 0 && phys < prm.num_blocks) {
              src_off = pool_row(phys, h, u_t0 % B, H, B, D);
              bytes = (uint32_t)rows * Tr::kRowBytes;
            } else {
              flag_error(PKV_DEV_BLOCK_ID);
            }
          }
        }
        uint32_t total = bytes;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        const bool load_q = (i == 0) && n_tok > 0;
        if (lane == 0) {
          int flags = done ? kTileEnd : ((i == 0 ? kTileFirst : 0) | (i == n_tiles - 1 ? kTileLast : 0));
          hdr[stage] = make_int4(s, h, p | (n_parts << 16), n_valid | (flags << 16));
          mbar_arrive_expect_tx(&full[stage], 2u * total + (load_q ? (uint32_t)Tr::kRowBytes : 0u));
        }
        __syncwarp();
        if (bytes) {
          unsigned char* st = smem + stage * Tr::kStageBytes + lane * unit_rows * Tr::kRowBytes;
          bulk_load(st, kc + src_off, bytes, &full[stage], policy);
          bulk_load(st + Tr::kTileBytes, vc + src_off, bytes, &full[stage], policy);
        }
        if (load_q && lane == 0) {
          bulk_load(smem + Tr::kQOffset + stage * Tr::kRowBytes, qg + ((size_t)s * H + h) * D, Tr::kRowBytes,
                    &full[stage], policy);
        }
      }
      if (done) break;
      u = __shfl_sync(0xffffffffu, u_next, 0);
    }
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

  float qf[Tr::kDimsPerLane];
  float acc[Tr::kDimsPerLane];
#pragma unroll
  for (int k = 0; k < Tr::kDimsPerLane; ++k) qf[k] = acc[k] = 0.f;
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
#pragma unroll
        for (int c = 0; c < Tr::kChunksPerLane; ++c) Elem<T>::widen(qrow[c * 8 + sub], qf + c * Tr::kPerChunk);
#pragma unroll
        for (int k = 0; k < Tr::kDimsPerLane; ++k) qf[k] *= prm.scale_log2;
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
          float f[Tr::kPerChunk];
          Elem<T>::widen(row[c * 8 + sub], f);
#pragma unroll
          for (int k = 0; k < Tr::kPerChunk; k += 2) {
            d0 = fmaf(qf[c * Tr::kPerChunk + k], f[k], d0);
            d1 = fmaf(qf[c * Tr::kPerChunk + k + 1], f[k + 1], d1);
          }
        }
      }
      float d = d0 + d1;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      d += __shfl_xor_sync(0xffffffffu, d, 4);
      x[j] = (r < n_valid) ? d : -INFINITY;
    }

    float mt = x[0];
#pragma unroll
    for (int j = 1; j < Tr::kTokPerGroup; ++j) mt = fmaxf(mt, x[j]);
    const float m_new = fmaxf(m, mt);
    if (m_new != -INFINITY) {
      const float alpha = exp2f(m - m_new);  // 0 while m is still -inf
      l *= alpha;
#pragma unroll
      for (int k = 0; k < Tr::kDimsPerLane; ++k) acc[k] *= alpha;
#pragma unroll
      for (int j = 0; j < Tr::kTokPerGroup; ++j) {
        const int r = j * Tr::kGroups + tok_lane;
        if (r < n_valid) {  // rows past the context are never read (they may hold NaN)
          const float pj = exp2f(x[j] - m_new);
          l += pj;
          const uint4* row = reinterpret_cast<const uint4*>(vt + r * Tr::kRowBytes);
#pragma unroll
          for (int c = 0; c < Tr::kChunksPerLane; ++c) {
            float f[Tr::kPerChunk];
            Elem<T>::widen(row[c * 8 + sub], f);
#pragma unroll
            for (int k = 0; k < Tr::kPerChunk; ++k)
              acc[c * Tr::kPerChunk + k] = fmaf(pj, f[k], acc[c * Tr::kPerChunk + k]);
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
    const int d = threadIdx.x;  // consumer thread d finalises dimension d
    if (d < D) {
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, rml[2 * w]);
      float L = 0.f, o = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float sc = (mx == -INFINITY) ? 0.f : exp2f(rml[2 * w] - mx);
        L = fmaf(rml[2 * w + 1], sc, L);
        o = fmaf(racc[w * D + d], sc, o);
      }
      const int us = hd.x, uh = hd.y, up = hd.z & 0xffff, un = hd.z >> 16;
      const size_t sh = (size_t)us * H + uh;
      if (un == 1) {
        prm.out[sh * D + d] = (L > 0.f) ? o / L : 0.f;
      } else {
        const size_t ws = sh * prm.max_parts + up;
        prm.ws_acc[ws * D + d] = o;
        if (d == 0) prm.ws_ml[ws] = make_float2(mx, L);
      }
    }
    ++units_done;
  }
}

// ---------------------------------------------------------------------------
// 3. log-sum-exp merge of the partitions of each (sequence, head):
//      M = max_p m_p,  L = sum_p l_p 2^(m_p - M),  out = sum_p acc_p 2^(m_p - M) / L.
//    Contexts that fit one partition were finished by the decode kernel.
//    grid = (num_heads, num_seqs); block = 128, thread d owns dimension d.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128)
    paged_decode_merge_kernel(const int32_t* __restrict__ context_lens, int num_heads, int max_ctx, int part_tokens,
                              int max_parts, const float* __restrict__ ws_acc, const float2* __restrict__ ws_ml,
                              float* __restrict__ out) {
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  const int np = parts_of(clamp_ctx(context_lens[s], max_ctx), part_tokens);
  if (np <= 1) return;
  const size_t sh = (size_t)s * num_heads + h;
  const size_t base = sh * max_parts;
  const int d = threadIdx.x;
  if (d >= D) return;
  float mx = -INFINITY;
  for (int p = 0; p < np; ++p) mx = fmaxf(mx, ws_ml[base + p].x);
  float L = 0.f, o = 0.f;
  for (int p = 0; p < np; ++p) {
    const float2 ml = ws_ml[base + p];
    const float sc = (mx == -INFINITY) ? 0.f : exp2f(ml.x - mx);
    L = fmaf(ml.y, sc, L);
    o = fmaf(ws_acc[(base + p) * D + d], sc, o);
  }
  out[sh * D + d] = (L > 0.f) ? o / L : 0.f;
}

}  // namespace pkv
