// cache_ops.cuh — KV-cache writes for sm_100a: slot mapping, reshape_and_cache
// (scatter new tokens into their slots) and copy_blocks (copy-on-write block
// duplication).  All three are bit copies / integer work with 16-byte vector
// accesses; at the sizes they run at (a few MB per call) they are bound by
// launch latency and one HBM round trip, not by bandwidth.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace pa {

// Slot of every new token: sequence s owns tokens [cu[s], cu[s+1]); token t
// sits at logical position ctx_lens[s] + t - cu[s]; its slot is
// block_tables[s][pos / B] * B + pos % B ("vLLM PagedAttention Deep Dive",
// "PagedAttention Mechanism").  cu == nullptr: one token per sequence.
__global__ void slot_mapping_kernel(int64_t* __restrict__ slots,
                                    const int32_t* __restrict__ block_tables,
                                    const int32_t* __restrict__ cu,
                                    const int32_t* __restrict__ ctx_lens, int num_seqs,
                                    int num_tokens, int max_blocks_per_seq, int block_size) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= num_tokens) return;
  int s = t, off = 0;
  if (cu != nullptr) {
    // last s with cu[s] <= t (binary search over the non-decreasing offsets)
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
    }
    s = lo;
    off = t - __ldg(cu + s);
  }
  const int pos = __ldg(ctx_lens + s) + off;
  const int blk = pos / block_size;
  if (pos < 0 || blk >= max_blocks_per_seq) {
    record_error(PA_DEVERR_SEQ_RANGE);
    slots[t] = -1;
    return;
  }
  const int phys = __ldg(block_tables + (size_t)s * max_blocks_per_seq + blk);
  slots[t] = (int64_t)phys * block_size + (pos % block_size);
}

// Slot of new token t: the slot-mapping rule above, shared by the fused
// append kernel (one thread per 16-byte chunk recomputes it; the table and
// lengths are tiny and cached).
__device__ __forceinline__ int64_t new_token_slot(const int32_t* __restrict__ block_tables,
                                                  const int32_t* __restrict__ cu,
                                                  const int32_t* __restrict__ ctx_lens,
                                                  int num_seqs, int t, int max_blocks_per_seq,
                                                  int block_size) {
  int s = t, off = 0;
  if (cu != nullptr) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
    }
    s = lo;
    off = t - __ldg(cu + s);
  }
  const int pos = __ldg(ctx_lens + s) + off;
  const int blk = pos / block_size;
  if (pos < 0 || blk >= max_blocks_per_seq) return -2;  // past the table
  return (int64_t)__ldg(block_tables + (size_t)s * max_blocks_per_seq + blk) * block_size +
         (pos % block_size);
}

// Fused append (slot mapping + reshape_and_cache in one launch): one thread
// per 16-byte chunk of one (token, kv head) row of K and of V; the first
// chunk of each token also stores its slot when `slots_out` is given.
template <int D>
__global__ void append_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                              uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                              const int32_t* __restrict__ block_tables,
                              const int32_t* __restrict__ cu, const int32_t* __restrict__ ctx_lens,
                              int64_t* __restrict__ slots_out, int num_seqs, int num_tokens,
                              int num_kv_heads, int max_blocks_per_seq, int block_size,
                              int num_blocks) {
  constexpr int CH = D * 2 / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * CH;
  if (idx >= total) return;
  const int c = (int)(idx % CH);
  const int64_t th = idx / CH;
  const int h = (int)(th % num_kv_heads);
  const int t = (int)(th / num_kv_heads);
  int64_t slot = new_token_slot(block_tables, cu, ctx_lens, num_seqs, t, max_blocks_per_seq,
                                block_size);
  const bool first = c == 0 && h == 0;
  if (slot == -2) {
    if (first) {
      record_error(PA_DEVERR_SEQ_RANGE);
      if (slots_out) slots_out[t] = -1;
    }
    return;
  }
  if (slot < 0 || slot >= (int64_t)num_blocks * block_size) {
    if (first) {
      record_error(PA_DEVERR_BLOCK_RANGE);
      if (slots_out) slots_out[t] = -1;
    }
    return;
  }
  if (first && slots_out) slots_out[t] = slot;
  const int64_t b = slot / block_size, off = slot % block_size;
  const int64_t dst = ((b * num_kv_heads + h) * block_size + off) * CH + c;
  const int64_t src = th * CH + c;
  const uint4 kv = __ldg(key + src);
  const uint4 vv = __ldg(value + src);
  key_cache[dst] = kv;
  value_cache[dst] = vv;
}

// One thread per 16-byte chunk of one (token, kv head) row of K and of V
// ("PagedAttention: KV cache as virtual memory", "Deep dive": a new token's
// K/V go into the next free slot of its sequence's last block).
template <int D>
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ key,
                                         const uint4* __restrict__ value,
                                         uint4* __restrict__ key_cache,
                                         uint4* __restrict__ value_cache,
                                         const int64_t* __restrict__ slot_mapping,
                                         int num_tokens, int num_kv_heads, int block_size,
                                         int64_t num_slots) {
  constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * CH;
  if (idx >= total) return;
  const int c = (int)(idx % CH);
  const int64_t th = idx / CH;  // token * Hkv + head
  const int h = (int)(th % num_kv_heads);
  const int64_t t = th / num_kv_heads;
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (c == 0) record_error(PA_DEVERR_SLOT_RANGE);
    return;
  }
  const int64_t b = slot / block_size, off = slot % block_size;
  const int64_t dst = ((b * num_kv_heads + h) * block_size + off) * CH + c;
  const int64_t src = th * CH + c;
  const uint4 kv = __ldg(key + src);
  const uint4 vv = __ldg(value + src);
  key_cache[dst] = kv;
  value_cache[dst] = vv;
}

// FP8 (E4M3) cache write: one thread per 16 elements of one (token, kv head)
// row of K and of V.  Each value is divided by its cache's scale in fp32
// (IEEE division) and rounded to the nearest E4M3 code, ties to even,
// magnitudes above 448 saturating ("PagedAttention: KV cache as virtual
// memory", "Interviewer follow-ups": an FP8 KV cache halves the bytes per
// block; the encoding and the per-cache scale are this library's reading).
// 16 consecutive fp16 / bf16 values at `in` (32-byte aligned) -> 16 E4M3
// codes of value / scale: IEEE fp32 division, nearest code with ties to even,
// saturation at +-448.
template <typename T>
__device__ __forceinline__ uint4 quantize16_e4m3(const T* in, float scale) {
  uint4 raw[2];
  raw[0] = __ldg(reinterpret_cast<const uint4*>(in));
  raw[1] = __ldg(reinterpret_cast<const uint4*>(in) + 1);
  const T* x = reinterpret_cast<const T*>(raw);
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(float(x[4 * q]) / scale, float(x[4 * q + 1]) / scale), __NV_SATFINITE,
        __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(float(x[4 * q + 2]) / scale, float(x[4 * q + 3]) / scale), __NV_SATFINITE,
        __NV_E4M3);
    w[q] = (lo & 0xFFFF) | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T>
__global__ void reshape_and_cache_fp8_kernel(const T* __restrict__ key, const T* __restrict__ value,
                                             uint8_t* __restrict__ key_cache,
                                             uint8_t* __restrict__ value_cache,
                                             const int64_t* __restrict__ slot_mapping,
                                             int num_tokens, int num_kv_heads, int head_dim,
                                             int block_size, int64_t num_slots, float k_scale,
                                             float v_scale) {
  const int CH = head_dim / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * CH;
  if (idx >= total) return;
  const int c = (int)(idx % CH);
  const int64_t th = idx / CH;  // token * Hkv + head
  const int h = (int)(th % num_kv_heads);
  const int64_t t = th / num_kv_heads;
  const int64_t slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (c == 0) record_error(PA_DEVERR_SLOT_RANGE);
    return;
  }
  const int64_t b = slot / block_size, off = slot % block_size;
  const int64_t src = th * head_dim + c * 16;
  const int64_t dst = ((b * num_kv_heads + h) * block_size + off) * head_dim + c * 16;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv)
    *reinterpret_cast<uint4*>((kv == 0 ? key_cache : value_cache) + dst) =
        quantize16_e4m3<T>((kv == 0 ? key : value) + src, kv == 0 ? k_scale : v_scale);
}

// Copy-on-write block copies ("PagedAttention: Why Static Batching Wastes
// Your KV Cache", "How does copy-on-write eliminate duplicate prompt KV
// cache?": the diverging sequence gets its own copy of just that block).
// One CTA per (pair, K-or-V); each thread moves kPerThread 16-byte chunks,
// all loads issued before the stores.
template <int kPerThread>
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                       const int64_t* __restrict__ pairs, int64_t chunks_per_block,
                       int num_blocks) {
  const int64_t src = __ldg(pairs + 2 * blockIdx.x), dst = __ldg(pairs + 2 * blockIdx.x + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0) record_error(PA_DEVERR_BLOCK_RANGE);
    return;
  }
  uint4* cache = blockIdx.y == 0 ? key_cache : value_cache;
  const uint4* from = cache + src * chunks_per_block;
  uint4* to = cache + dst * chunks_per_block;
  for (int64_t base = 0; base < chunks_per_block; base += (int64_t)kPerThread * 256) {
    uint4 r[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int64_t i = base + (int64_t)k * 256 + threadIdx.x;
      if (i < chunks_per_block) r[k] = from[i];
    }
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int64_t i = base + (int64_t)k * 256 + threadIdx.x;
      if (i < chunks_per_block) to[i] = r[k];
    }
  }
}

// Block copies between two pools (swap out to / in from host memory;
// "PagedAttention: Why Static Batching Wastes Your KV Cache", "What happens
// when the GPU runs out of KV blocks?").  One
// CTA per (pair, K-or-V); either pool may be pinned host memory mapped into
// the GPU's address space, so the loads or the stores cross PCIe / C2C; all
// of a thread's loads are issued before its stores to keep many in flight.
template <int kPerThread>
__global__ void __launch_bounds__(256)
    swap_blocks_kernel(uint4* dst_k, uint4* dst_v, const uint4* src_k, const uint4* src_v,
                       const int64_t* __restrict__ pairs, int64_t chunks_per_block,
                       int src_blocks, int dst_blocks) {
  const int64_t src = pairs[2 * blockIdx.x], dst = pairs[2 * blockIdx.x + 1];
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (threadIdx.x == 0) record_error(PA_DEVERR_BLOCK_RANGE);
    return;
  }
  const uint4* from = (blockIdx.y == 0 ? src_k : src_v) + src * chunks_per_block;
  uint4* to = (blockIdx.y == 0 ? dst_k : dst_v) + dst * chunks_per_block;
  for (int64_t base = 0; base < chunks_per_block; base += (int64_t)kPerThread * 256) {
    uint4 r[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int64_t i = base + (int64_t)k * 256 + threadIdx.x;
      if (i < chunks_per_block) r[k] = from[i];
    }
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int64_t i = base + (int64_t)k * 256 + threadIdx.x;
      if (i < chunks_per_block) to[i] = r[k];
    }
  }
}

}  // namespace pa
