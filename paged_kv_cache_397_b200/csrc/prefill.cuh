// prefill.cuh — causal chunked-prefill attention against the paged context,
// on the sm_100a tcgen05 tensor cores.
//
// What it computes ("vLLM PagedAttention Deep Dive", "Mechanics of Chunked
// Prefill" and "PagedAttention Mechanism"): chunk query i of sequence s
// (absolute position ctx_lens[s] + i) attends, with standard softmax
// attention, to the logical tokens 0 .. ctx_lens[s] + i of its KV head, read
// through block_tables[s]; the chunk's own K/V are already in the cache.
//
// How (B200 design, one CTA per (128-query tile, query head, sequence)):
//  * warp 4 (TMA): loads the Q tile once and streams 128-token K and V tiles
//    into a 2-stage ring.  A tile is gathered block by block: each logical
//    block is one TMA box per 64 columns at row (phys * Hkv + kvh) * B of the
//    pool viewed as a 2-D [rows, head_dim] tensor, 128-byte swizzled, so the
//    gather needs no address arithmetic on the compute warps.
//  * warp 5 (MMA, one thread): S_j = Q K_j^T with tcgen05.mma (M=128, N=128,
//    K=16 steps, both operands K-major in shared memory) into one of two
//    128-column TMEM buffers; then O += P_{j-1} V_{j-1} with P read from
//    tensor memory and V as an MN-major shared-memory operand.  Completion is
//    signalled with tcgen05.commit on mbarriers.
//  * warps 0-3 (softmax): thread r owns query row r = TMEM lane r.  It loads
//    its S row with tcgen05.ld, applies the causal / length mask, keeps a
//    running max that is only raised when the tile max exceeds it by more
//    than 2^8 (so O is rescaled in TMEM rarely; the stale max cancels in
//    O / l), writes P = exp2(S - m) as 16-bit values over the S buffer with
//    tcgen05.st, and finally divides O by the row sum and stores the row.
//  * V rows past the end of the sequence (unwritten slots, NaN allowed) are
//    zeroed in shared memory before their PV product.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace pa {

struct PrefillParams {
  void* out;  // T[total_q][Hq][D]
  const int32_t* block_tables;
  const int32_t* cu_q_lens;
  const int32_t* ctx_lens;
  int num_seqs, total_q, num_q_heads, num_kv_heads, group;
  int num_blocks, max_blocks_per_seq;
  float scale_log2;
};

template <typename T, int BS>
struct PrefillShape {
  static constexpr int D = 128;
  static constexpr int BM = 128;                // query rows per CTA
  static constexpr int BN = 128;                // keys per tile
  static constexpr int THREADS = 6 * 32;
  static constexpr int HALF = BM * 128;         // one 64-column group of a 128-row tile (16 KB)
  static constexpr int TILE = 2 * HALF;         // 128 x 128 x 2 bytes = 32 KB
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE;            // 2 stages
  static constexpr int V_OFF = 3 * TILE;        // 2 stages
  static constexpr int BAR_OFF = 5 * TILE;
  static constexpr int NBAR = 16;
  static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NBAR * 8 + 16;
  static constexpr int BLOCKS_PER_TILE = BN / BS;
  static constexpr uint32_t TMEM_COLS = 512;    // S0 | S1 | O | (unused)
};

template <typename T, int BS>
__global__ void __launch_bounds__(PrefillShape<T, BS>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
  using Sh = PrefillShape<T, BS>;
  constexpr int D = Sh::D, BM = Sh::BM, BN = Sh::BN;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;  // [2]
  uint64_t* o_done = bars + 13;
  uint64_t* o_final = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Sh::NBAR);

  const int qtile = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = p.cu_q_lens[s];
  const int n = p.cu_q_lens[s + 1] - q0;
  const int i0 = qtile * BM;
  if (i0 >= n) return;
  const int c = p.ctx_lens[s];
  int L = c + n;  // tokens in the cache for this sequence
  if (L > p.max_blocks_per_seq * BS) {
    if (threadIdx.x == 0 && h == 0 && qtile == 0) record_error(PA_DEVERR_SEQ_RANGE);
    L = p.max_blocks_per_seq * BS;
  }
  const int kvh = h / p.group;
  const int rows = min(BM, n - i0);
  // keys needed by the last row of this tile (bounded by the sequence length)
  const int kv_end = min(L, c + i0 + rows);
  const int ntiles = (kv_end + BN - 1) / BN;
  const int nblk_seq = (L + BS - 1) / BS;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Sh::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s[2] = {tmem, tmem + 128};
  const uint32_t t_o = tmem + 256;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA warp
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, Sh::TILE);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_2d(smem + Sh::Q_OFF + hf * Sh::HALF, &tm_q, h * D + hf * 64, q0 + i0, q_full,
                    pol_q);
    }
    const int32_t* bt = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    bool alive = true;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j & 1;
      const int b0 = j * Sh::BLOCKS_PER_TILE;
      const int nb = min(Sh::BLOCKS_PER_TILE, nblk_seq - b0);
      int phys = 0;
      if (lane < nb) {
        phys = __ldg(bt + b0 + lane);
        if (phys < 0 || phys >= p.num_blocks) {
          record_error(PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
      }
      const uint32_t bytes = (uint32_t)nb * BS * D * 2;
      if (lane == 0) {
        if (j >= 2 && alive) alive = mbar_wait(&k_empty[st], ((j >> 1) - 1) & 1);
        mbar_arrive_expect_tx(&k_full[st], bytes);
      }
      for (int b = 0; b < nb; ++b) {
        const int ph = __shfl_sync(0xffffffffu, phys, b);
        if (lane == 0) {
          const int row = (ph * p.num_kv_heads + kvh) * BS;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(smem + Sh::K_OFF + st * Sh::TILE + hf * Sh::HALF + b * BS * 128, &tm_k,
                        hf * 64, row, &k_full[st], pol_kv);
        }
      }
      if (lane == 0) {
        if (j >= 2 && alive) alive = mbar_wait(&v_empty[st], ((j >> 1) - 1) & 1);
        mbar_arrive_expect_tx(&v_full[st], bytes);
      }
      for (int b = 0; b < nb; ++b) {
        const int ph = __shfl_sync(0xffffffffu, phys, b);
        if (lane == 0) {
          const int row = (ph * p.num_kv_heads + kvh) * BS;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(smem + Sh::V_OFF + st * Sh::TILE + hf * Sh::HALF + b * BS * 128, &tm_v,
                        hf * 64, row, &v_full[st], pol_kv);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA warp
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(128, 128, kBf16, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(128, 128, kBf16, false, true);
      const uint32_t sq = smem_u32(smem + Sh::Q_OFF);
      bool alive = mbar_wait(q_full, 0);
      tc_fence_after();
      for (int j = 0; j <= ntiles; ++j) {
        if (j < ntiles) {
          const int st = j & 1;
          if (alive) alive = mbar_wait(&k_full[st], (j >> 1) & 1);
          tc_fence_after();
          const uint32_t sk = smem_u32(smem + Sh::K_OFF + st * Sh::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * Sh::HALF + (kk & 3) * 32;
            umma_ss(t_s[st], umma_desc_sw128(sq + off, 16, 1024),
                    umma_desc_sw128(sk + off, 16, 1024), idesc_qk, kk > 0);
          }
          umma_commit(&s_full[st]);
          umma_commit(&k_empty[st]);
        }
        if (j >= 1) {
          const int jp = j - 1, st = jp & 1;
          if (alive) alive = mbar_wait(&p_full[st], (jp >> 1) & 1);
          if (alive) alive = mbar_wait(&v_full[st], (jp >> 1) & 1);
          tc_fence_after();
          const uint32_t sv = smem_u32(smem + Sh::V_OFF + st * Sh::TILE);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            umma_ts(t_o, t_s[st] + kk * 8, umma_desc_sw128(sv + kk * 16 * 128, Sh::HALF, 1024),
                    idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&v_empty[st]);
          umma_commit(o_done);
          if (j == ntiles) umma_commit(o_final);
        }
      }
    }
  } else {
    // -------------------------------------------------------- softmax warps
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int qpos = c + i0 + r;                // absolute position of this row's query
    const int limit = min(qpos, L - 1);         // last visible key
    float m_run = -INFINITY, l_run = 0.f;
    bool alive = true;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j & 1;
      if (alive) alive = mbar_wait(&s_full[st], (j >> 1) & 1);
      tc_fence_after();
      if (j == ntiles - 1 && L - j * BN < BN) {
        // Zero V rows past the sequence end before the last PV product.  S_j
        // complete implies PV_{j-2} complete, hence this V stage's previous
        // use has landed and the parity below names the current phase (a
        // wait on an older phase could alias the next, never-completing one).
        if (alive) alive = mbar_wait(&v_full[st], (j >> 1) & 1);
        const int first = L - j * BN;
        uint8_t* sv = smem + Sh::V_OFF + st * Sh::TILE;
        for (int idx = r; idx < (BN - first) * 16; idx += 128) {
          const int row = first + idx / 16, ch = idx % 16;
          *reinterpret_cast<uint4*>(sv + (ch >> 3) * Sh::HALF + row * 128 + (ch & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      float sv[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t rr[32];
        tmem_ld32(t_s[st] + lane_off + cc * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[cc * 32 + e] = __uint_as_float(rr[e]);
      }
      const int kbase = j * BN;
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; ++e) {
        const float x = (kbase + e <= limit) ? sv[e] * p.scale_log2 : -INFINITY;
        sv[e] = x;
        mx = fmaxf(mx, x);
      }
      if (mx > m_run + 8.0f) {
        // raise the running max; rescale l and O (O only exists after tile 0)
        const float alpha = exp2f(m_run - mx);
        l_run *= alpha;
        if (j > 0) {
          if (alive) alive = mbar_wait(o_done, (j - 1) & 1);
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t rr[32];
            tmem_ld32(t_o + lane_off + cc * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st32(t_o + lane_off + cc * 32, rr);
          }
        }
        m_run = mx;
      }
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = exp2f(sv[cc * 32 + 2 * e] - m_run);
          const float b = exp2f(sv[cc * 32 + 2 * e + 1] - m_run);
          rs += a + b;
          pk[e] = MmaOp<T>::pack(a, b);
        }
        tmem_st16(t_s[st] + lane_off + cc * 16, pk);
      }
      l_run += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[st]);
    }
    // epilogue: O / l for the valid rows, once the last PV product is done
    // (a one-shot barrier, so the wait cannot alias another phase).
    if (alive) alive = mbar_wait(o_final, 0);
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(q0 + i0 + r) * p.num_q_heads + h) * D;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t rr[32];
      tmem_ld32(t_o + lane_off + cc * 32, rr);
      tmem_wait_ld();
      if (r < rows) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = MmaOp<T>::pack(__uint_as_float(rr[2 * e]) * inv,
                                 __uint_as_float(rr[2 * e + 1]) * inv);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          reinterpret_cast<uint4*>(orow + cc * 32)[v] =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::TMEM_COLS);
  }
}

}  // namespace pa
