// prefill.cuh — causal chunked-prefill attention against the paged context,
// on the sm_100a tcgen05 tensor cores.
//
// What it computes ("vLLM PagedAttention Deep Dive", "Mechanics of Chunked
// Prefill" and "PagedAttention Mechanism"): chunk query i of sequence s
// (absolute position ctx_lens[s] + i) attends, with standard softmax
// attention, to the logical tokens 0 .. ctx_lens[s] + i of its KV head, read
// through block_tables[s]; the chunk's own K/V are already in the cache.
//
// How (B200 design).  One CTA per (256 chunk rows, query head, sequence); the
// 256 rows are two 128-row Q tiles that share every K/V tile:
//  * warp 8 (TMA): loads both Q tiles once, then streams K_0, V_0, K_1, V_1,
//    ... through a 4-stage shared-memory ring.  A 128-token tile is gathered
//    block by block — one TMA box per block per 64 columns at row
//    (phys * Hkv + kvh) * B of the pool viewed as a 2-D [rows, head_dim]
//    tensor, 128-byte swizzled — with the boxes of a tile issued in parallel
//    by the warp's lanes.
//  * warp 9 (MMA, one thread): tcgen05.mma kind::f16, fp32 accumulation in
//    tensor memory.  S_w = Q_w K_j^T (M=128, N=128, K-major operands in
//    shared memory) and O_w += P_w V_j (P from tensor memory, V an MN-major
//    shared-memory operand).  Issue order: S0_0, S1_0, then for every tile
//    PV0_j, S0_{j+1}, PV1_j, S1_{j+1}: while one softmax warpgroup works on
//    its scores, the tensor core runs the other tile's products.  PV_w(j)
//    goes out in two parts: its first 4 K-steps (keys 0-63) once the softmax
//    warps report that part of P stored, the rest with P complete.
//    Completion is signalled with tcgen05.commit on mbarriers.
//  * warps 0-3 and 4-7 (softmax, one warpgroup per Q tile): thread r owns
//    query row r = TMEM lane r.  It loads its S row (tcgen05.ld), masks only
//    on tiles that reach past its causal limit, keeps a running max raised
//    only when a tile's max exceeds it by more than 2^8 (the stale max
//    cancels in O / l, so O in tensor memory is rarely rescaled), writes
//    P = exp2(S * scale - m) as 16-bit values over its S columns (tcgen05.st),
//    and finally stores O / l.  Because S_w(j) is issued after PV_w(j-1),
//    "S_w(j) complete" already implies O_w is up to date for a rescale.
//  * V rows past the end of the sequence (unwritten slots, NaN allowed) are
//    zeroed in shared memory by warpgroup 0 before the last PV products.
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
  // Work units (one per 256 chunk rows of a query head of a sequence) in
  // launch order; units [n_full, ...) are tail units whose KV range is cut
  // into `split` parts (split == 1: none).
  int tiles_per_seq;  // 256-row tiles per sequence (from the host's max_q_len)
  int n_full;
  int split;
  float* ws_o;        // [tail parts][D / 4][256] float4: unnormalised O of each part
  float* ws_ml;       // [tail parts][256][2] (running max in log2 units, sum)
  int* counters;      // [tail units] parts finished; zero at launch
};

template <typename T, int BS, int D_ = 128>
struct PrefillShape {
  static constexpr int D = D_;                  // head_dim: 64 or 128
  static constexpr int NH = D / 64;             // 64-column (128-byte) halves of a row
  static constexpr int BM = 128;                // rows per Q tile
  static constexpr int NQ = 2;                  // Q tiles per CTA
  static constexpr int BN = 128;                // keys per K/V tile
  static constexpr int THREADS = 12 * 32;       // 3 warpgroups
  static constexpr int TMA_WARP = 8, MMA_WARP = 9;  // warps 10-11 idle
  // Registers per thread after setmaxnreg: softmax warpgroups grow, the
  // producer warpgroup shrinks.  2*128*200 + 128*96 = 63488 must not exceed
  // the launch allocation THREADS * MIN_LAUNCH_REGS = 64512, so the host
  // refuses to launch a build whose kernel has fewer than MIN_LAUNCH_REGS.
  static constexpr uint32_t SOFTMAX_REGS = 200, PRODUCER_REGS = 96;
  static constexpr int MIN_LAUNCH_REGS = 168;
  static_assert(2 * 128 * SOFTMAX_REGS + 128 * PRODUCER_REGS <= THREADS * MIN_LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static constexpr int HALF = 128 * 128;        // 128 rows x 64 columns x 2 bytes
  static constexpr int TILE = NH * HALF;        // 128 rows x D columns x 2 bytes (16 or 32 KB)
  // K/V ring stages (K_j, V_j alternate): the same 128 KB at either head_dim
  static constexpr int NSTAGE = 4 * (2 / NH);
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NQ * TILE;
  static constexpr int BAR_OFF = RING_OFF + NSTAGE * TILE;
  static constexpr int NBAR = 1 + 2 * NSTAGE + 4 * NQ + 1;  // + the MMA drain barrier
  static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NBAR * 8 + 16;
  static constexpr int BLOCKS_PER_TILE = BN / BS;
  static constexpr uint32_t TMEM_COLS = 512;    // S0 | S1 | O0 | O1 (O: D columns of 128)
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(NH * BLOCKS_PER_TILE <= 32, "one TMA box per lane");
};

// S_w = Q_w K^T: D / 16 K-steps of 16 over head_dim, both operands K-major,
// SW128 (steps 4-7 in the second 64-column half, HALF bytes on).
template <int HALF, int D>
__device__ __forceinline__ void prefill_issue_s(uint32_t d_tmem, uint32_t q_smem,
                                                uint32_t k_smem, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
    umma_ss(d_tmem, umma_desc_sw128(q_smem + off, 16, 1024),
            umma_desc_sw128(k_smem + off, 16, 1024), idesc, kk > 0);
  }
}

// O_w += P_w V over the K-steps [K0, K1) of 16 keys; P from tensor memory (8
// columns of packed 16-bit pairs per step), V MN-major with its two 64-column
// halves HALF bytes apart.
template <int HALF, int K0, int K1>
__device__ __forceinline__ void prefill_issue_pv(uint32_t o_tmem, uint32_t p_tmem,
                                                 uint32_t v_smem, uint32_t idesc, bool first) {
#pragma unroll
  for (int kk = K0; kk < K1; ++kk)
    umma_ts(o_tmem, p_tmem + kk * 8, umma_desc_sw128(v_smem + kk * 16 * 128, HALF, 1024), idesc,
            (!first || kk > 0) ? 1u : 0u);
}

// KV-split tail unit, after this part's partial rows are stored (O as
// [part][D / 4][256 rows] float4, so a warp's stores and loads are
// contiguous; (m, l) as [part][256 rows][2]): the 256 softmax threads (row =
// thread) count the part in; the part that completes the count combines all
// parts of the unit in part order, so the result does not depend on which
// part finishes last:
//   M = max_q m_q,  o = sum_q 2^(m_q - M) O_q / sum_q 2^(m_q - M) l_q.
template <typename T, int D>
__device__ __forceinline__ void prefill_combine_tail(const PrefillParams& p, int slot, int row,
                                                     bool row_valid, T* orow, int* flag) {
  __threadfence();
  named_barrier(2, 256);
  if (threadIdx.x == 0) *flag = atomicAdd(&p.counters[slot], 1) == p.split - 1;
  named_barrier(2, 256);
  if (!*flag) return;
  __threadfence();
  const size_t base = (size_t)slot * p.split;
  float mq[4], M = -INFINITY;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    mq[q] = q < p.split ? __ldcg(p.ws_ml + ((base + q) * 256 + row) * 2) : -INFINITY;
    M = fmaxf(M, mq[q]);
  }
  const float m_use = M == -INFINITY ? 0.f : M;
  float sc[4], den = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    sc[q] = q < p.split ? exp2f(mq[q] - m_use) : 0.f;
    if (q < p.split) den += sc[q] * __ldcg(p.ws_ml + ((base + q) * 256 + row) * 2 + 1);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  if (!row_valid) return;
  const float4* ws4 = reinterpret_cast<const float4*>(p.ws_o);
  constexpr int C = 4;  // float4 per chunk: 16 columns, all parts' loads in flight together
#pragma unroll 1
  for (int v0 = 0; v0 < D / 4; v0 += C) {
    float4 part_rows[4][C];  // the other parts' columns, loaded together
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int c = 0; c < C; ++c)
        if (q < p.split)
          part_rows[q][c] = __ldcg(ws4 + ((base + q) * (D / 4) + v0 + c) * 256 + row);
    float acc[4 * C];
#pragma unroll
    for (int e = 0; e < 4 * C; ++e) acc[e] = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q >= p.split) continue;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const float4 x = part_rows[q][c];
        acc[4 * c] += sc[q] * x.x;
        acc[4 * c + 1] += sc[q] * x.y;
        acc[4 * c + 2] += sc[q] * x.z;
        acc[4 * c + 3] += sc[q] * x.w;
      }
    }
    uint32_t pk[2 * C];
#pragma unroll
    for (int e = 0; e < 2 * C; ++e) pk[e] = MmaOp<T>::pack(acc[2 * e] * inv, acc[2 * e + 1] * inv);
#pragma unroll
    for (int c = 0; c < C / 2; ++c)
      reinterpret_cast<uint4*>(orow + 4 * v0)[c] =
          make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  }
}

// P = 2^(S * scale - m) for the 16-column chunks [C0, C1) of a softmax
// thread's S row (in sv), written as 16-bit pairs over the row's S columns in
// tensor memory (P of chunk cc goes to columns 8 cc .. 8 cc + 7, which the
// thread has already read), with the row sum of P accumulated in four packed
// fp32 partial sums.
template <typename T, int C0, int C1>
__device__ __forceinline__ void prefill_p_chunks(const uint32_t (&sv)[128], uint64_t sc2,
                                                 uint64_t negm2, uint32_t t_s,
                                                 uint64_t (&rsum)[4]) {
#pragma unroll
  for (int cc = C0; cc < C1; ++cc) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int x = cc * 16 + 2 * e;
      float a, b;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[x]), __uint_as_float(sv[x + 1])), sc2, negm2),
                a, b);
      a = ex2_approx(a);
      b = ex2_approx(b);
      rsum[e & 3] = f2_add(rsum[e & 3], f2_pack(a, b));
      pk[e] = MmaOp<T>::pack(a, b);
    }
    tmem_st8(t_s + cc * 8, pk);
  }
}

// The work of one CTA: chunk rows tile * 256 .. tile * 256 + 255 of query
// head h of sequence s, over the whole causal key range (nparts == 1) or over
// part `part` of it, split into nparts runs of 128-key tiles (tail unit
// `slot`; the parts' partial rows are combined by the last one to finish).
// Needs every thread of the CTA (12 warps, or more: warps past the producer
// warpgroup idle), 1024-byte aligned shared memory at `smem` and all 512
// tensor-memory columns.  SOFT_REGS / PROD_REGS / IDLE_REGS: the setmaxnreg
// split between the two softmax warpgroups, the producer warpgroup and any
// warpgroup past it.
template <typename T, int BS, uint32_t SOFT_REGS = PrefillShape<T, BS>::SOFTMAX_REGS,
          uint32_t PROD_REGS = PrefillShape<T, BS>::PRODUCER_REGS, int HEAD_DIM = 128,
          uint32_t IDLE_REGS = PROD_REGS>
__device__ __forceinline__ void prefill_tile(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                             const CUtensorMap* tm_v, const PrefillParams& p,
                                             uint8_t* smem, int tile, int h, int s, int part = 0,
                                             int nparts = 1, int slot = 0) {
  using Sh = PrefillShape<T, BS, HEAD_DIM>;
  constexpr int D = Sh::D, BM = Sh::BM, BN = Sh::BN, NQ = Sh::NQ, NS = Sh::NSTAGE;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::BAR_OFF);
  uint64_t* q_full = bars;                        // 1
  uint64_t* ring_full = bars + 1;                 // NS
  uint64_t* ring_empty = bars + 1 + NS;           // NS
  uint64_t* s_full = bars + 1 + 2 * NS;           // NQ
  uint64_t* p_full = s_full + NQ;                 // NQ
  uint64_t* o_final = p_full + NQ;                // NQ
  uint64_t* p_half = o_final + NQ;                // NQ: P of the tile's first 64 keys
  uint64_t* mma_drain = p_half + NQ;              // 1 (used only after an abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Sh::NBAR);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(last_flag + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = p.cu_q_lens[s];
  const int n = p.cu_q_lens[s + 1] - q0;
  const int i0 = tile * (NQ * BM);  // first chunk row of this CTA
  if (i0 >= n) return;
  const int c = p.ctx_lens[s];
  int L = c + n;  // tokens in the cache for this sequence
  if (L > p.max_blocks_per_seq * BS) {
    if (threadIdx.x == 0 && h == 0 && tile == 0) record_error(PA_DEVERR_SEQ_RANGE);
    L = p.max_blocks_per_seq * BS;
  }
  const int kvh = h / p.group;
  const int rows = min(NQ * BM, n - i0);            // valid rows of this CTA
  const int kv_end = min(L, c + i0 + rows);         // keys the last valid row needs
  const int ntiles_all = (kv_end + BN - 1) / BN;    // >= 1
  const int j0 = part * ntiles_all / nparts;         // this part's key tiles [j0, j1)
  const int ntiles = (part + 1) * ntiles_all / nparts - j0;
  const int nblk_seq = (L + BS - 1) / BS;
  if (ntiles == 0) {
    // an empty part of a split unit (fewer key tiles than parts): it counts
    // in with an empty partial, and may be the one that combines
    if (warp >= 8) return;
    const int r = threadIdx.x;  // row of the CTA's 256
    const size_t u = (size_t)slot * p.split + part;
    p.ws_ml[(u * 256 + r) * 2] = -INFINITY;
    p.ws_ml[(u * 256 + r) * 2 + 1] = 0.f;
    float4* dst = reinterpret_cast<float4*>(p.ws_o) + u * (D / 4) * 256 + r;
    for (int v = 0; v < D / 4; ++v) dst[v * 256] = make_float4(0.f, 0.f, 0.f, 0.f);
    prefill_combine_tail<T, D>(p, slot, r, i0 + r < n,
                               reinterpret_cast<T*>(p.out) +
                                   ((size_t)(q0 + i0 + r) * p.num_q_heads + h) * D,
                               last_flag);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1);
    }
    for (int w = 0; w < NQ; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], 4);  // one arrival per softmax warp
      mbar_init(&p_half[w], 4);
      mbar_init(&o_final[w], 1);
    }
    mbar_init(mma_drain, 1);
    *abort = 0;
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

  int armed = 0;  // TMA warp: ring items (K_j = 2j, V_j = 2j + 1) armed so far
  if (warp >= 12) {
    // warpgroups past the producer warpgroup (a CTA of the mixed launch): idle
    setmaxnreg_dec<IDLE_REGS>();
  } else if (warp >= 8) {
    // producer warpgroup: TMA warp, MMA warp, two idle warps
    setmaxnreg_dec<PROD_REGS>();
  if (warp == Sh::TMA_WARP) {
    // ------------------------------------------------------------ TMA warp
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(tm_q);
      tma_prefetch_desc(tm_k);
      tma_prefetch_desc(tm_v);
      mbar_arrive_expect_tx(q_full, NQ * Sh::TILE);
    }
    __syncwarp();
    if (lane < Sh::NH * NQ) {  // lane -> (Q tile, 64-column half)
      const int w = lane / Sh::NH, hf = lane % Sh::NH;
      tma_load_2d(smem + Sh::Q_OFF + w * Sh::TILE + hf * Sh::HALF, tm_q, h * D + hf * 64,
                  q0 + i0 + w * BM, q_full, pol_q);
    }
    const int32_t* bt = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    for (int j = 0; j < ntiles && armed == 2 * j; ++j) {
      const int b0 = (j0 + j) * Sh::BLOCKS_PER_TILE;
      const int nb = min(Sh::BLOCKS_PER_TILE, nblk_seq - b0);
      int phys = 0;
      if (lane < nb) {
        phys = __ldg(bt + b0 + lane);
        if (phys < 0 || phys >= p.num_blocks) {
          record_error(PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
      }
      // lane l issues the box of block l / NH, 64-column half l % NH
      const int ph = __shfl_sync(0xffffffffu, phys, (lane / Sh::NH) & 31);
      const int row = (ph * p.num_kv_heads + kvh) * BS;
      const uint32_t bytes = (uint32_t)nb * BS * D * 2;
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int item = 2 * j + kv, st = item % NS;
        int ok = 1;
        if (lane == 0) {
          if (item >= NS) ok = mbar_wait(&ring_empty[st], ((item / NS) - 1) & 1, abort);
          if (ok) mbar_arrive_expect_tx(&ring_full[st], bytes);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;  // gave up: load nothing more
        if (lane < Sh::NH * nb) {
          const int hf = lane % Sh::NH;
          tma_load_2d(smem + Sh::RING_OFF + st * Sh::TILE + hf * Sh::HALF +
                          (lane / Sh::NH) * BS * 128,
                      kv == 0 ? tm_k : tm_v, hf * 64, row, &ring_full[st], pol_kv);
        }
        armed = item + 1;
      }
    }
  } else if (warp == Sh::MMA_WARP) {
    // ------------------------------------------------------------ MMA warp
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(128, 128, kBf16, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(128, D, kBf16, false, true);
      const uint32_t sq = smem_u32(smem + Sh::Q_OFF);
      const uint32_t ring = smem_u32(smem + Sh::RING_OFF);
      bool alive = mbar_wait(q_full, 0, abort) && mbar_wait(&ring_full[0], 0, abort);  // Q, K_0
      if (alive) {
        tc_fence_after();
        prefill_issue_s<Sh::HALF, D>(tmem, sq, ring, idesc_qk);
        umma_commit(&s_full[0]);
        prefill_issue_s<Sh::HALF, D>(tmem + 128, sq + Sh::TILE, ring, idesc_qk);
        umma_commit(&s_full[1]);
        umma_commit(&ring_empty[0]);
      }
      for (int j = 0; alive && j < ntiles; ++j) {
        const int it_v = 2 * j + 1, st_v = it_v % NS;
        const int it_k = 2 * j + 2, st_k = it_k % NS;
        const bool more = j + 1 < ntiles;
        // V_j and K_{j+1} first: they are normally in shared memory long
        // before P0_j, so nothing but P stands between a softmax hand-off and
        // the next products
        if (!mbar_wait(&ring_full[st_v], (it_v / NS) & 1, abort)) break;
        if (more && !mbar_wait(&ring_full[st_k], (it_k / NS) & 1, abort)) break;
        // tile 0: PV0_j over the first 64 keys as soon as their P is
        // written, the rest with P complete, then S0_{j+1}
        if (!mbar_wait(&p_half[0], j & 1, abort)) break;
        tc_fence_after();
        prefill_issue_pv<Sh::HALF, 0, 4>(tmem + 256, tmem, ring + st_v * Sh::TILE, idesc_pv,
                                         j == 0);
        if (!mbar_wait(&p_full[0], j & 1, abort)) break;
        tc_fence_after();
        prefill_issue_pv<Sh::HALF, 4, 8>(tmem + 256, tmem, ring + st_v * Sh::TILE, idesc_pv,
                                         false);
        if (more) {
          prefill_issue_s<Sh::HALF, D>(tmem, sq, ring + st_k * Sh::TILE, idesc_qk);
          umma_commit(&s_full[0]);
        } else {
          umma_commit(&o_final[0]);
        }
        // tile 1: PV1_j in the same two parts, then S1_{j+1}
        if (!mbar_wait(&p_half[1], j & 1, abort)) break;
        tc_fence_after();
        prefill_issue_pv<Sh::HALF, 0, 4>(tmem + 384, tmem + 128, ring + st_v * Sh::TILE,
                                         idesc_pv, j == 0);
        if (!mbar_wait(&p_full[1], j & 1, abort)) break;
        tc_fence_after();
        prefill_issue_pv<Sh::HALF, 4, 8>(tmem + 384, tmem + 128, ring + st_v * Sh::TILE,
                                         idesc_pv, false);
        umma_commit(&ring_empty[st_v]);
        if (more) {
          prefill_issue_s<Sh::HALF, D>(tmem + 128, sq + Sh::TILE, ring + st_k * Sh::TILE, idesc_qk);
          umma_commit(&s_full[1]);
          umma_commit(&ring_empty[st_k]);
        } else {
          umma_commit(&o_final[1]);
        }
      }
    }
  }
  } else {
    // -------------------------------------------------- softmax warpgroups
    setmaxnreg_inc<SOFT_REGS>();
    const int w = warp >> 2;                       // Q tile of this warpgroup
    const int r = threadIdx.x & 127;               // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + w * 128;
    const uint32_t t_o = tmem + lane_base + 256 + w * 128;
    const int row = i0 + w * BM + r;               // chunk row of this thread
    const int limit = min(c + row, L - 1);         // last key this row may see
    const float sc = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;          // running max in log2 units
    bool alive = true;
    for (int j = 0; j < ntiles; ++j) {
      // after a wait gave up every lane runs on through its (garbage) tiles
      // alike, so the .aligned tensor-memory accesses stay converged
      if (alive) alive = mbar_wait(&s_full[w], j & 1, abort);
      tc_fence_after();
      const int kbase = (j0 + j) * BN;
      if (w == 0 && j == ntiles - 1 && L - kbase < BN) {
        // Zero V rows past the sequence end before PV0/PV1 of the last tile.
        // S0_j complete implies every earlier use of V_j's stage landed, so
        // this parity names the current phase.
        const int it_v = 2 * j + 1, st_v = it_v % NS;
        if (alive) alive = mbar_wait(&ring_full[st_v], (it_v / NS) & 1, abort);
        const int first = L - kbase;
        uint8_t* vs = smem + Sh::RING_OFF + st_v * Sh::TILE;
        constexpr int CH = D / 8;  // 16-byte chunks per row
        for (int idx = r; idx < (BN - first) * CH; idx += 128) {
          const int vr = first + idx / CH, ch = idx % CH;
          *reinterpret_cast<uint4*>(vs + (ch >> 3) * Sh::HALF + vr * 128 + (ch & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      uint32_t sv[BN];
      tmem_ld32_at<0>(t_s, sv);
      tmem_ld32_at<32>(t_s + 32, sv);
      tmem_ld32_at<64>(t_s + 64, sv);
      tmem_ld32_at<96>(t_s + 96, sv);
      tmem_wait_ld();
      if (kbase + BN - 1 > limit) {  // only tiles that reach past this row's limit
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (kbase + e > limit) sv[e] = __float_as_uint(-INFINITY);
      }
      // row max: four independent chains of three-input max
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < BN; e += 8) {
        mx[0] = fmax3(mx[0], __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
        mx[1] = fmax3(mx[1], __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
        mx[2] = fmax3(mx[2], __uint_as_float(sv[e + 4]), __uint_as_float(sv[e + 5]));
        mx[3] = fmax3(mx[3], __uint_as_float(sv[e + 6]), __uint_as_float(sv[e + 7]));
      }
      const float m_tile = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;  // scale > 0 commutes
      // The running max is raised only when the tile max exceeds it by more
      // than 8 (log2 units): P <= 2^8 stays in 16-bit range and O is rarely
      // rescaled (the stale max cancels in O / l).
      const bool raise = m_tile > m_run + 8.0f;
      float alpha = 1.f;
      if (raise) {
        alpha = exp2f(m_run - m_tile);  // 0 while m_run is -inf
        l_run *= alpha;
        m_run = m_tile;
      }
      // rescale O (S_w(j) complete implies PV_w(j-1) complete), 32 columns at
      // a time, the S row staying live in registers; warp-uniform (the
      // tensor-memory accesses are .aligned): rows whose max is unchanged
      // multiply by 1
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(t_o + cc * 32, ov);
          tmem_wait_ld_into<0>(ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(t_o + cc * 32, ov);
        }
      }
      // P = 2^(S * scale - m): packed FMA, SFU exp2, packed row sums.  A row
      // with no visible key yet (only in a later part of a split unit) keeps
      // m_run = -inf: use 0 so that its masked scores give 0.
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      uint64_t rsum[4] = {0, 0, 0, 0};  // four packed partial row sums of P
      const uint64_t sc2 = f2_pack(sc, sc), negm2 = f2_pack(-m_use, -m_use);
      prefill_p_chunks<T, 0, BN / 32>(sv, sc2, negm2, t_s, rsum);
      // the first 64 keys' P (columns 0-31) goes to the MMA thread while the
      // rest is computed
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&p_half[w]);
      prefill_p_chunks<T, BN / 32, BN / 16>(sv, sc2, negm2, t_s, rsum);
      float l0, l1;
      f2_unpack(f2_add(f2_add(rsum[0], rsum[1]), f2_add(rsum[2], rsum[3])), l0, l1);
      l_run += l0 + l1;
      // hand P to the MMA thread: every lane's stores are complete and ordered
      // before the warp's one arrival
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&p_full[w]);
    }
    // epilogue: O / l for the valid rows (one-shot barrier per Q tile)
    if (alive) alive = mbar_wait(&o_final[w], 0, abort);
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(q0 + row) * p.num_q_heads + h) * D;
    uint32_t ov[D];
    tmem_ld32_at<0>(t_o, ov);
    tmem_ld32_at<32>(t_o + 32, ov);
    if constexpr (D == 128) {
      tmem_ld32_at<64>(t_o + 64, ov);
      tmem_ld32_at<96>(t_o + 96, ov);
    }
    tmem_wait_ld();
    if (nparts == 1) {
      if (row < n) {
#pragma unroll
        for (int v = 0; v < D / 8; ++v) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pk[e] = MmaOp<T>::pack(__uint_as_float(ov[8 * v + 2 * e]) * inv,
                                   __uint_as_float(ov[8 * v + 2 * e + 1]) * inv);
          reinterpret_cast<uint4*>(orow)[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    } else {
      // partial row of this part: unnormalised O, running max, sum
      const int rr = w * BM + r;  // row of the CTA's 256
      const size_t u = (size_t)slot * p.split + part;
      float4* dst = reinterpret_cast<float4*>(p.ws_o) + u * (D / 4) * 256 + rr;
#pragma unroll
      for (int v = 0; v < D / 4; ++v)
        dst[v * 256] = make_float4(__uint_as_float(ov[4 * v]), __uint_as_float(ov[4 * v + 1]),
                                   __uint_as_float(ov[4 * v + 2]), __uint_as_float(ov[4 * v + 3]));
      p.ws_ml[(u * 256 + rr) * 2] = m_run;
      p.ws_ml[(u * 256 + rr) * 2 + 1] = l_run;
      prefill_combine_tail<T, D>(p, slot, rr, row < n, orow, last_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort) {
    // a wait gave up: let this CTA's own loads and tensor-core products land
    // before its shared and tensor memory are released
    if (warp == Sh::TMA_WARP && lane == 0) {
      mbar_drain(q_full, 0);
      drain_ring<NS>(ring_full, armed);
    }
    if (warp == Sh::MMA_WARP && lane == 0) {
      umma_commit(mma_drain);
      mbar_drain(mma_drain, 0);
    }
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Sh::TMEM_COLS);
  }
}

template <typename T, int BS, int D>
__global__ void __launch_bounds__(PrefillShape<T, BS, D>::THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // 1-D grid: units in launch order, tail units' parts last
  const int b = blockIdx.x;
  int unit = b, part = 0, nparts = 1, slot = 0;
  if (b >= p.n_full) {
    slot = (b - p.n_full) / p.split;
    part = (b - p.n_full) % p.split;
    nparts = p.split;
    unit = p.n_full + slot;
  }
  const int tile = unit % p.tiles_per_seq;
  const int h = (unit / p.tiles_per_seq) % p.num_q_heads;
  const int s = unit / (p.tiles_per_seq * p.num_q_heads);
  prefill_tile<T, BS, PrefillShape<T, BS, D>::SOFTMAX_REGS, PrefillShape<T, BS, D>::PRODUCER_REGS,
               D>(&tm_q, &tm_k, &tm_v, p, smem, tile, h, s, part, nparts, slot);
}

}  // namespace pa
