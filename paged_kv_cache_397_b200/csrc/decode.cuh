// decode.cuh — paged decode attention for sm_100a.
//
// What it computes ("vLLM PagedAttention Deep Dive", "PagedAttention
// Mechanism"): for every sequence s and query head h, softmax attention of the
// single query row q[s][h] over the first seq_lens[s] logical tokens of KV
// head h / G, whose K/V rows are gathered through block_tables[s].
//
// How (B200 design):
//  * One CTA per (split-KV partition, KV head, sequence).  A partition is a
//    fixed run of logical blocks, so the work split and every reduction order
//    depend only on logical positions (bit-identical results under any
//    relabelling of physical blocks) and long sequences fill all 148 SMs.
//  * GQA: the CTA reads each (block, KV head) K/V tile from HBM exactly once
//    and applies it to all G query heads of the group.
//  * One producer warp streams the (block, KV head) tiles — each a
//    contiguous block_size x head_dim run of the pool — into a ring of shared
//    memory stages with TMA (cp.async.bulk.tensor, 128-byte swizzle, one
//    16-byte-aligned box per 64 columns), completing on mbarriers.  The
//    block-table entries of a partition are fetched once, coalesced, by the
//    producer warp.
//  * Four consumer warps take blocks round-robin.  Each 16-token sub-tile is
//    a tiny GEMM pair on the warp-level tensor-core path (mma.sync m16n8k16,
//    fp32 accumulate): S^T = K Q^T puts tokens on M and the (padded) query
//    heads on N; P^T is moved into the B-operand layout in registers with
//    movmatrix; O^T += V^T P^T reads V transposed with ldmatrix.trans.  Online
//    softmax (running max, exp2, rescale) stays in registers; the max uses
//    warp shuffles.  Decode is HBM-bound, so the point of the tensor path is
//    only to keep ALU issue far below the memory time.
//  * Warps merge their softmax states in shared memory in a fixed order.  A
//    sequence with one partition writes the final row; otherwise the
//    partition writes (m, l, acc) to the workspace and decode_reduce_kernel
//    combines partitions with the log-sum-exp rule in partition order.
#pragma once

#include "ptx.cuh"

namespace pa {

struct DecodeParams {
  void* out;                 // T[S][Hq][D]
  const void* query;         // T[S][Hq][D]
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* ws_acc;             // [S][Hq][max_parts][D]
  float* ws_ml;              // [S][Hq][max_parts][2]  (m in log2 units, l)
  int num_seqs, num_q_heads, num_kv_heads, group;
  int num_blocks, max_blocks_per_seq;
  int part_blocks;           // logical blocks per partition
  int max_parts;             // gridDim.x
  float scale_log2;          // softmax scale * log2(e)
};

template <typename T, int D, int BS, int NT>
struct DecodeShape {
  static constexpr int NW = 4;                      // consumer warps
  static constexpr int THREADS = (NW + 1) * 32;     // + producer warp
  static constexpr int HALVES = D / 64;             // 128-byte column groups
  static constexpr int HALF_BYTES = BS * 128;       // one column group of a tile
  static constexpr int TILE_BYTES = BS * D * 2;     // K or V tile of one (block, kv head)
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = (BS == 16) ? 8 : 4;     // ring depth
  static constexpr int RING_BYTES = NS * STAGE_BYTES;
  static constexpr int MERGE_BYTES = NW * (NT * 8) * (D + 2) * 4;
  static constexpr int BODY_BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
  static constexpr int SMEM_BYTES = 1024 + BODY_BYTES + 2 * NS * 8;
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(BS == 16 || BS == 32, "block_size");
  static_assert(NS % NW == 0 || NW % NS == 0, "ring depth vs consumer warps");
};

template <typename T, int D, int BS, int NT>
__global__ void __launch_bounds__(DecodeShape<T, D, BS, NT>::THREADS, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, DecodeParams p) {
  using Shape = DecodeShape<T, D, BS, NT>;
  constexpr int NW = Shape::NW, NS = Shape::NS, HALVES = Shape::HALVES;
  constexpr int GP = NT * 8;  // padded heads per CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Shape::BODY_BYTES);
  uint64_t* empty_bar = full_bar + NS;

  const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // A length beyond the table or beyond the launch's partitions (max_seq_len)
  // is a caller error: flag it and attend over the tokens that fit.
  int L = p.seq_lens[s];
  const int L_cap = min(p.max_blocks_per_seq, p.max_parts * p.part_blocks) * BS;
  if (L > L_cap) {
    if (threadIdx.x == 0 && part == 0 && kvh == 0) record_error(PA_DEVERR_SEQ_RANGE);
    L = L_cap;
  }
  if (L < 0) L = 0;
  const int nblk_seq = (L + BS - 1) / BS;
  const int nparts = nblk_seq == 0 ? 1 : (nblk_seq + p.part_blocks - 1) / p.part_blocks;
  if (part >= nparts) return;
  const int blk0 = part * p.part_blocks;
  const int nblk = min(p.part_blocks, nblk_seq - blk0);  // 0 only when L == 0

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const uint64_t policy = l2_policy_evict_first();
    const int32_t* bt = p.block_tables + (size_t)s * p.max_blocks_per_seq + blk0;
    bool alive = true;
    for (int base = 0; base < nblk; base += 32) {
      int phys = 0;
      if (base + lane < nblk) {
        phys = __ldg(bt + base + lane);
        if (phys < 0 || phys >= p.num_blocks) {
          record_error(PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
      }
      const int cnt = min(32, nblk - base);
      for (int j = 0; j < cnt; ++j) {
        const int ph = __shfl_sync(0xffffffffu, phys, j);
        if (lane == 0) {
          const int i = base + j, st = i % NS;
          if (i >= NS && alive) alive = mbar_wait(&empty_bar[st], ((i / NS) - 1) & 1);
          mbar_arrive_expect_tx(&full_bar[st], Shape::STAGE_BYTES);
          uint8_t* sk = smem + st * Shape::STAGE_BYTES;
          uint8_t* sv = sk + Shape::TILE_BYTES;
          const int row = (ph * p.num_kv_heads + kvh) * BS;
#pragma unroll
          for (int h = 0; h < HALVES; ++h) {
            tma_load_2d(sk + h * Shape::HALF_BYTES, &tm_k, h * 64, row, &full_bar[st], policy);
            tma_load_2d(sv + h * Shape::HALF_BYTES, &tm_v, h * 64, row, &full_bar[st], policy);
          }
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int G = p.group;
  const int c4 = lane & 3, r4 = lane >> 2;
  // Q^T as the B operand (k = head dim, n = query head of the group).
  uint32_t qf[D / 16][NT][2];
  {
    const T* qbase = reinterpret_cast<const T*>(p.query) +
                     ((size_t)s * p.num_q_heads + (size_t)kvh * G) * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + r4;
#pragma unroll
      for (int kt = 0; kt < D / 16; ++kt) {
        uint32_t b0 = 0, b1 = 0;
        if (g < G) {
          const uint32_t* row = reinterpret_cast<const uint32_t*>(qbase + (size_t)g * D);
          b0 = __ldg(row + (kt * 16 + 2 * c4) / 2);
          b1 = __ldg(row + (kt * 16 + 2 * c4 + 8) / 2);
        }
        qf[kt][nt][0] = b0;
        qf[kt][nt][1] = b1;
      }
    }
  }

  float m_run[NT][2], l_run[NT][2];
  float o[D / 16][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[dt][nt][e] = 0.f;
  }

  const uint32_t smem_base = smem_u32(smem);
  bool alive = true;
  for (int i = warp; i < nblk; i += NW) {
    const int st = i % NS;
    if (alive) alive = mbar_wait(&full_bar[st], (i / NS) & 1);
    const uint32_t sk = smem_base + st * Shape::STAGE_BYTES;
    const uint32_t sv = sk + Shape::TILE_BYTES;
    const int tok_blk = (blk0 + i) * BS;  // logical position of the block's first slot
    const int valid = min(BS, L - tok_blk);
    if (valid < BS) {
      // Slots past the sequence end may hold anything (NaN included); zero
      // their V rows so that 0-weight x garbage cannot poison the PV product.
      uint8_t* v_gen = smem + st * Shape::STAGE_BYTES + Shape::TILE_BYTES;
      for (int idx = lane; idx < (BS - valid) * HALVES * 8; idx += 32) {
        const int r = valid + idx / (HALVES * 8), rem = idx % (HALVES * 8);
        const int h = rem / 8, ch = rem % 8;
        *reinterpret_cast<uint4*>(v_gen + h * Shape::HALF_BYTES + r * 128 + ch * 16) =
            make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
#pragma unroll
    for (int mt = 0; mt < BS / 16; ++mt) {
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
      // S^T = K Q^T
#pragma unroll
      for (int kt = 0; kt < D / 16; ++kt) {
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = (kt & 3) * 2 + (lane >> 4);
        const uint32_t addr = sk + (kt >> 2) * Shape::HALF_BYTES + row * 128 +
                              ((chunk ^ (row & 7)) << 4);
        uint32_t a[4];
        ldmatrix_x4(a, addr);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) MmaOp<T>::run(sacc[nt], a, qf[kt][nt][0], qf[kt][nt][1]);
      }
      // online softmax over this sub-tile's 16 tokens
      const int t_lo = tok_blk + mt * 16 + r4;
      const bool ok_lo = t_lo < L, ok_hi = t_lo + 8 < L;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float pv[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float s_lo = ok_lo ? sacc[nt][j] * p.scale_log2 : -INFINITY;
          const float s_hi = ok_hi ? sacc[nt][j + 2] * p.scale_log2 : -INFINITY;
          float mx = fmaxf(s_lo, s_hi);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][j], mx);
          const float m_use = m_new == -INFINITY ? 0.f : m_new;
          const float alpha = exp2f(m_run[nt][j] - m_use);
          pv[j] = exp2f(s_lo - m_use);
          pv[j + 2] = exp2f(s_hi - m_use);
          l_run[nt][j] = l_run[nt][j] * alpha + pv[j] + pv[j + 2];
          m_run[nt][j] = m_new;
#pragma unroll
          for (int dt = 0; dt < D / 16; ++dt) {
            o[dt][nt][j] *= alpha;
            o[dt][nt][j + 2] *= alpha;
          }
        }
        // accumulator rows t / t+8, cols (g, g+1) -> B-operand layout of P^T
        pb[nt][0] = movmatrix_trans(MmaOp<T>::pack(pv[0], pv[1]));
        pb[nt][1] = movmatrix_trans(MmaOp<T>::pack(pv[2], pv[3]));
      }
      // O^T += V^T P^T
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        const int j = lane >> 3;
        const int trow = mt * 16 + (lane & 7) + (j >> 1) * 8;
        const int dcol = dt * 16 + (j & 1) * 8;
        const int chunk = (dcol & 63) >> 3;
        const uint32_t addr = sv + (dcol >> 6) * Shape::HALF_BYTES + trow * 128 +
                              ((chunk ^ (trow & 7)) << 4);
        uint32_t a[4];
        ldmatrix_x4_trans(a, addr);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) MmaOp<T>::run(o[dt][nt], a, pb[nt][0], pb[nt][1]);
      }
    }
    if (valid < BS) fence_proxy_async_smem();  // our zero stores precede the next TMA write
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);
  }

  // ------------------------------------------------- merge the 4 warp states
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][j] = l;
    }
  named_barrier(1, NW * 32);  // every consumer is done reading the ring
  float* mg = reinterpret_cast<float*>(smem);  // [NW][GP][D + 2]: acc[D], m, l
  constexpr int RS = D + 2;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = dt * 16 + r4 + (e >> 1) * 8;
        const int g = nt * 8 + 2 * c4 + (e & 1);
        mg[(warp * GP + g) * RS + d] = o[dt][nt][e];
      }
  if (r4 == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int g = nt * 8 + 2 * c4 + j;
        mg[(warp * GP + g) * RS + D] = m_run[nt][j];
        mg[(warp * GP + g) * RS + D + 1] = l_run[nt][j];
      }
  }
  named_barrier(1, NW * 32);
  const bool single = (nparts == 1);
  for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
    const int g = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mg[(w * GP + g) * RS + D]);
    const float m_use = M == -INFINITY ? 0.f : M;
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float sc = exp2f(mg[(w * GP + g) * RS + D] - m_use);
      num += sc * mg[(w * GP + g) * RS + d];
      den += sc * mg[(w * GP + g) * RS + D + 1];
    }
    const int h = kvh * G + g;
    if (single) {
      const float v = den > 0.f ? num / den : 0.f;
      reinterpret_cast<T*>(p.out)[((size_t)s * p.num_q_heads + h) * D + d] = T(v);
    } else {
      const size_t row = ((size_t)s * p.num_q_heads + h) * p.max_parts + part;
      p.ws_acc[row * D + d] = num;
      if (d == 0) {
        p.ws_ml[row * 2] = M;
        p.ws_ml[row * 2 + 1] = den;
      }
    }
  }
}

// Log-sum-exp combine of split-KV partitions, in partition order.  One CTA
// of D threads per (sequence, query head); sequences that fit one partition
// were finished by decode_kernel and are skipped.
template <typename T, int D>
__global__ void __launch_bounds__(D)
    decode_reduce_kernel(DecodeParams p, int block_size) {
  const int s = blockIdx.x / p.num_q_heads, h = blockIdx.x % p.num_q_heads;
  int L = p.seq_lens[s];
  L = max(0, min(L, min(p.max_blocks_per_seq, p.max_parts * p.part_blocks) * block_size));
  const int nblk = (L + block_size - 1) / block_size;
  const int nparts = nblk == 0 ? 1 : (nblk + p.part_blocks - 1) / p.part_blocks;
  if (nparts <= 1) return;
  const size_t row0 = ((size_t)s * p.num_q_heads + h) * p.max_parts;
  const int d = threadIdx.x;
  float M = -INFINITY;
  for (int q = 0; q < nparts; ++q) M = fmaxf(M, p.ws_ml[(row0 + q) * 2]);
  const float m_use = M == -INFINITY ? 0.f : M;
  float num = 0.f, den = 0.f;
  for (int q = 0; q < nparts; ++q) {
    const float sc = exp2f(p.ws_ml[(row0 + q) * 2] - m_use);
    num += sc * p.ws_acc[(row0 + q) * D + d];
    den += sc * p.ws_ml[(row0 + q) * 2 + 1];
  }
  const float v = den > 0.f ? num / den : 0.f;
  reinterpret_cast<T*>(p.out)[((size_t)s * p.num_q_heads + h) * D + d] = T(v);
}

}  // namespace pa
