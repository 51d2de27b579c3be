// Cache-maintenance kernels: per-token append into slots, copy-on-write block
// copy, and a contiguous gather of one sequence.  All three are pure data
// movement in 16-byte vectors; the copies are bit-exact.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// kv_cache_append: grid = (num_tokens, 2 for K|V); the CTA of token t copies its
// num_heads rows of row_vecs 16-byte vectors into the slot's rows (one per head).
constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_cache,
                     uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int num_heads,
                     int row_vecs, int block_size, long long num_slots) {
  // a programmatic dependent (the decode plan) may start now: it reads nothing
  // this kernel writes, and waits for it to complete before its own writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = blockIdx.x;
  const int is_v = blockIdx.y;
  const long long slot = slot_mapping[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (is_v == 0 && threadIdx.x == 0) flag_error(PKV_DEV_SLOT);
    return;
  }
  const long long blk = slot / block_size;
  const int off = (int)(slot - blk * block_size);
  const int per_token = num_heads * row_vecs;
  const uint4* src = (is_v ? v_new : k_new) + (size_t)t * per_token;
  uint4* cache = is_v ? v_cache : k_cache;
  for (int i = threadIdx.x; i < per_token; i += kAppendThreads) {
    const int h = i / row_vecs;
    const int vec = i - h * row_vecs;
    cache[pool_row(blk, h, off, num_heads, block_size, row_vecs) + vec] = src[i];
  }
}

// kv_block_copy: grid = (chunks per block, num_pairs, 2 for K|V); each thread moves
// kCopyVecs 16-byte vectors, all loads issued before the stores.
constexpr int kCopyThreads = 256;
constexpr int kCopyVecs = 4;

__global__ void __launch_bounds__(kCopyThreads)
    kv_block_copy_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                         const int64_t* __restrict__ pairs, long long block_vecs, int num_blocks) {
  const long long src = pairs[2 * (size_t)blockIdx.y];
  const long long dst = pairs[2 * (size_t)blockIdx.y + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(PKV_DEV_COPY_PAIR);
    return;
  }
  uint4* pool = blockIdx.z ? v_cache : k_cache;
  const uint4* from = pool + (size_t)src * block_vecs;
  uint4* to = pool + (size_t)dst * block_vecs;
  const long long base = (long long)blockIdx.x * (kCopyThreads * kCopyVecs) + threadIdx.x;
  uint4 buf[kCopyVecs];
#pragma unroll
  for (int j = 0; j < kCopyVecs; ++j) {
    const long long idx = base + (long long)j * kCopyThreads;
    if (idx < block_vecs) buf[j] = from[idx];
  }
#pragma unroll
  for (int j = 0; j < kCopyVecs; ++j) {
    const long long idx = base + (long long)j * kCopyThreads;
    if (idx < block_vecs) to[idx] = buf[j];
  }
}

// kv_blocks_to_host / kv_blocks_from_host: grid = (chunks per block, blocks, 2 for K|V).
// Slot i of the host buffers is block ids[i] of the pool; the host side is pinned
// memory reached through its device address (loads or stores cross the host link).
__global__ void __launch_bounds__(kCopyThreads)
    kv_swap_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, uint4* __restrict__ host_k,
                   uint4* __restrict__ host_v, const int64_t* __restrict__ ids, long long block_vecs, int num_blocks,
                   int to_host) {
  const long long b = ids[blockIdx.y];
  if (b < 0 || b >= num_blocks) {
    if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(PKV_DEV_COPY_PAIR);
    return;
  }
  uint4* pool = (blockIdx.z ? v_cache : k_cache) + (size_t)b * block_vecs;
  uint4* host = (blockIdx.z ? host_v : host_k) + (size_t)blockIdx.y * block_vecs;
  const uint4* from = to_host ? pool : host;
  uint4* to = to_host ? host : pool;
  const long long base = (long long)blockIdx.x * (kCopyThreads * kCopyVecs) + threadIdx.x;
  uint4 buf[kCopyVecs];
#pragma unroll
  for (int j = 0; j < kCopyVecs; ++j) {
    const long long idx = base + (long long)j * kCopyThreads;
    if (idx < block_vecs) buf[j] = from[idx];
  }
#pragma unroll
  for (int j = 0; j < kCopyVecs; ++j) {
    const long long idx = base + (long long)j * kCopyThreads;
    if (idx < block_vecs) to[idx] = buf[j];
  }
}

// paged_kv_gather: out[h][t][:] = cache[table[t / B]][h][t % B][:].  Rows are
// addressed with pool_row, the helper the decode kernel's producer uses.
__global__ void __launch_bounds__(256)
    kv_gather_kernel(const uint4* __restrict__ cache, const int32_t* __restrict__ table, int context_len,
                     int num_heads, int row_vecs, int block_size, int num_blocks, uint4* __restrict__ out) {
  const long long total = (long long)num_heads * context_len * row_vecs;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(i / ((long long)context_len * row_vecs));
    long long r = i - (long long)h * context_len * row_vecs;
    const int t = (int)(r / row_vecs);
    const int vec = (int)(r - (long long)t * row_vecs);
    const int phys = table[t / block_size];
    if (phys < 0 || phys >= num_blocks) {
      if (vec == 0) flag_error(PKV_DEV_BLOCK_ID);
      continue;
    }
    const size_t src = pool_row(phys, h, t % block_size, num_heads, block_size, row_vecs) + vec;
    out[i] = cache[src];
  }
}

}  // namespace pkv
