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
//  * The (block, KV head) tiles — each a contiguous block_size x head_dim
//    run of the pool — stream into a ring of shared-memory stages with TMA
//    (cp.async.bulk.tensor, 128-byte swizzle, boxes starting on 16-byte
//    boundaries), completing on mbarriers.  A producer warp issues the first
//    ring positions (and writes the step's new token first, when the append
//    is fused); from then on each consumer warp refills the stage it has
//    just consumed with its own next position there, so no stage waits
//    behind another warp's (item_ring_init / item_ring_fill / consume_item).
//  * Four consumer warps take blocks round-robin.  Each 16-token sub-tile is
//    a tiny GEMM pair on the warp-level tensor-core path (mma.sync m16n8k16,
//    fp32 accumulate): S^T = K Q^T puts tokens on M and the (padded) query
//    heads on N; P^T is moved into the B-operand layout in registers with
//    movmatrix; O^T += V^T P^T.  Online softmax (running max, exp2, rescale)
//    stays in registers; the max uses warp shuffles.  Decode is HBM-bound, so
//    the point of the tensor path is only to keep ALU issue far below the
//    memory time.
//  * Warps merge their softmax states in shared memory in a fixed order.  A
//    sequence with one partition writes the final row; otherwise the
//    partition writes (m, l, acc) to the workspace and decode_reduce_kernel
//    combines partitions with the log-sum-exp rule in partition order.
//
// Two cache formats share that skeleton through a tile policy:
//  * HalfTiles — fp16 / bf16 caches; K and V^T fragments come from the
//    swizzled tiles through ldmatrix / ldmatrix.trans; MMA in the cache type.
//  * E4m3Tiles — FP8 (E4M3) caches with one scale per cache ("PagedAttention:
//    KV cache as virtual memory", "Interviewer follow-ups": FP8 KV halves the
//    bytes per block).  K fragments come from 16-byte shared loads, V^T
//    fragments from ldmatrix .m16n16 .trans .b8 (the tokens of a sub-tile in
//    the order that load gives, K's rows loaded in the same order), both
//    converted e4m3x2 -> f16x2; MMA in fp16 (the query is rounded to fp16;
//    E4M3 values are exact in fp16).  k_scale is folded into the softmax scale
//    and v_scale multiplies the output once.
#pragma once

#include <cuda_fp8.h>

#include "cache_ops.cuh"
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
  float scale_log2;          // softmax scale * log2(e) (FP8: also * k_scale)
  float v_scale;             // FP8: multiplies the output; 1 otherwise
  float k_scale;             // FP8 with the fused append: the K cache's scale
  int len_add;               // tokens attended = seq_lens[s] + len_add (mixed batch: 1)
  // Fused append (pa_append_decode; null otherwise): the new token of
  // sequence s, at logical position seq_lens[s], is written into the cache
  // by the CTAs of its last partition before they read that block.
  const void* new_key;       // T[S][Hkv][D]
  const void* new_value;     // T[S][Hkv][D]
  void* key_cache;           // T[num_blocks][Hkv][BS][D] (FP8: E4M3 codes)
  void* value_cache;
  int64_t* slot_out;         // [S] slot written (-1: none), or null
  // Shared-prefix decode (pa_decode_shared_prefix): partition blockIdx.x of a
  // launch is partition part_base + blockIdx.x of the sequence; the prefix
  // launch reads the shared blocks from prefix_blocks and serves seq_group
  // sequences per CTA.
  int part_base = 0;
  const int32_t* prefix_blocks = nullptr;
  int seq_group = 1;
};

// ------------------------------------------------------------------ tiles
// Address of byte `col` of row `row` in a tile of 128-byte rows written by a
// TMA box with 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int col) {
  return base + row * 128 + ((((col >> 4) ^ (row & 7)) << 4) | (col & 15));
}

// fp16 / bf16 cache: a (block, kv head) tile is BS rows x D columns, stored as
// D/64 column groups of BS x 128 bytes.
template <typename T, int D_, int BS>
struct HalfTiles {
  using Elem = T;   // query / output type
  using MmaT = T;   // MMA operand type
  static constexpr int D = D_;
  static constexpr int BOXES = D / 64;              // TMA boxes per tile
  static constexpr int BOX_BYTES = BS * 128;
  static constexpr int HP = 1;                       // KV heads per ring stage
  static constexpr bool kHalfCache = true;           // cache elements are T
  static constexpr int TILE_ROWS = BS;               // one cache block per ring stage
  static constexpr int TILE_BYTES = BS * D * 2;
  static constexpr int NS = BS == 16 ? 8 : 4;        // ring depth
  static constexpr int NW = 4;                       // consumer warps per CTA
  // resident CTAs per SM to plan registers for, by query n-tiles per CTA
  static constexpr int min_ctas(int nt) { return nt == 1 ? 3 : 2; }
  static constexpr int ZERO_CHUNKS_PER_ROW = BOXES * 8;

  // K and V of the cache block at pool row `row` into block slot u (always 0)
  __device__ static void issue(uint8_t* sk, uint8_t* sv, const CUtensorMap* mk,
                               const CUtensorMap* mv, int row, int /*u*/, uint64_t* bar,
                               uint64_t pol) {
#pragma unroll
    for (int h = 0; h < BOXES; ++h) {
      tma_load_2d(sk + h * BOX_BYTES, mk, h * 64, row, bar, pol);
      tma_load_2d(sv + h * BOX_BYTES, mv, h * 64, row, bar, pol);
    }
  }
  // 16-byte chunk `idx` of V row `r` (for zeroing rows past the sequence end)
  __device__ static uint8_t* zero_chunk(uint8_t* v, int r, int idx) {
    return v + (idx >> 3) * BOX_BYTES + r * 128 + (idx & 7) * 16;
  }
  // Q^T as the B operand: k = head dim in natural order; query column g
  // (g < G) is the row qbase + g * D
  template <int NT>
  __device__ static void load_q(uint32_t (&qf)[D / 16][NT][2], const T* qbase, int G,
                                int lane) {
    load_q_cols<NT>(qf, [&](int g) { return g < G ? qbase + (size_t)g * D : nullptr; }, lane);
  }
  // the same with column g taken from row_of(g) (nullptr: a zero column)
  template <int NT, class RowOf>
  __device__ static void load_q_cols(uint32_t (&qf)[D / 16][NT][2], RowOf row_of, int lane) {
    const int c4 = lane & 3, r4 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + r4;
      const T* qrow = row_of(g);
#pragma unroll
      for (int kt = 0; kt < D / 16; ++kt) {
        uint32_t b0 = 0, b1 = 0;
        if (qrow != nullptr) {
          const uint32_t* row = reinterpret_cast<const uint32_t*>(qrow);
          b0 = __ldg(row + (kt * 16 + 2 * c4) / 2);
          b1 = __ldg(row + (kt * 16 + 2 * c4 + 8) / 2);
        }
        qf[kt][nt][0] = b0;
        qf[kt][nt][1] = b1;
      }
    }
  }
  // S^T (16 tokens of sub-tile mt x 8*NT heads) = K Q^T
  template <int NT>
  __device__ static void qk(float (&sacc)[NT][4], const uint8_t* tile, int mt,
                            const uint32_t (&qf)[D / 16][NT][2], int lane) {
    qk_at<NT>(sacc, smem_u32(tile), mt, qf, lane);
  }
  template <int NT>
  __device__ static void qk_at(float (&sacc)[NT][4], uint32_t sk, int mt,
                            const uint32_t (&qf)[D / 16][NT][2], int lane) {
    float acc2[NT][4];  // odd k-steps accumulate separately (two shorter MMA chains)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc2[nt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < D / 16; ++kt) {
      const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int chunk = (kt & 3) * 2 + (lane >> 4);
      const uint32_t addr = sk + (kt >> 2) * BOX_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4);
      uint32_t a[4];
      ldmatrix_x4(a, addr);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        MmaOp<MmaT>::run((kt & 1) ? acc2[nt] : sacc[nt], a, qf[kt][nt][0], qf[kt][nt][1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] += acc2[nt][e];
  }
  // O^T (D x 8*NT) += V^T P^T for sub-tile mt
  template <int NT>
  __device__ static void pv(float (&o)[D / 16][NT][4], const uint8_t* tile, int mt,
                            const uint32_t (&pb)[NT][2], int lane) {
    pv_at<NT>(o, smem_u32(tile), mt, pb, lane);
  }
  template <int NT>
  __device__ static void pv_at(float (&o)[D / 16][NT][4], uint32_t sv, int mt,
                            const uint32_t (&pb)[NT][2], int lane) {
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      const int j = lane >> 3;
      const int trow = mt * 16 + (lane & 7) + (j >> 1) * 8;
      const int dcol = dt * 16 + (j & 1) * 8;
      const int chunk = (dcol & 63) >> 3;
      const uint32_t addr =
          sv + (dcol >> 6) * BOX_BYTES + trow * 128 + ((chunk ^ (trow & 7)) << 4);
      uint32_t a[4];
      ldmatrix_x4_trans(a, addr);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) MmaOp<MmaT>::run(o[dt][nt], a, pb[nt][0], pb[nt][1]);
    }
  }
  // head-dim index of accumulator element o[dt][.][e] of lane row r4
  __device__ static int out_d(int dt, int e, int r4) { return dt * 16 + r4 + (e >> 1) * 8; }
  // S^T accumulator rows r4 and r4 + 8 of a 16-row sub-tile hold tokens
  // row_lo(r4) and row_lo(r4) + HI_STEP of the sub-tile
  __device__ static int row_lo(int r4) { return r4; }
  static constexpr int HI_STEP = 8;
};

// FP8 E4M3 cache, head_dim 128: a tile is BS rows x 128 bytes (one TMA box).
// Q K^T contracts over the head dim in the permuted order d = 32c + 4kt + j
// (c = lane % 4, kt = k-step, j = 0..3), so lane c reads bytes [32c, 32c+32)
// of a K row with two 16-byte loads.  O^T keeps head-dim rows in the permuted
// order d = 16r + 4p + b (r = lane / 4, p = m-tile pair, b = byte), so the
// V^T fragments of a 16-token sub-tile come from one 16-byte load per token
// row; byte_perm pairs two token rows along the contraction (token) axis.
template <typename T, int BS, int HP_ = 1>
struct E4m3Tiles {
  using Elem = T;
  using MmaT = __half;
  static constexpr int D = 128;
  static constexpr int BOXES = 1;
  // A ring stage is a 32-row tile of 128-byte rows whatever the cache block
  // size, and each consumer warp has two stages in flight.  With 16-token
  // blocks it holds either HP = 2 adjacent KV heads of one block (one
  // contiguous 4 KB box: the two heads' 2 x G query heads fill the 8-wide MMA
  // n-tile, each head's columns masked to its own rows) or, when the group
  // is too wide for that, two blocks of one head (two 2 KB boxes; each starts
  // on a 1 KB swizzle atom, so the stage reads like one 32-row tile).  On
  // B200 the FP8 path is latency bound: two 16-row sub-tiles per stage and
  // two stages per warp (8 stages, 3 CTAs per SM) stream 5.4 TB/s with
  // 32-token blocks, against 4.6 TB/s for one 16-token block per stage at
  // four CTAs per SM and 3.5 TB/s for 32-token blocks with 4 stages.
  static constexpr int HP = HP_;
  static constexpr bool kHalfCache = false;  // cache elements are E4M3 codes
  static constexpr int BOX_BYTES = HP * BS * 128;
  static constexpr int TILE_ROWS = 32;
  static constexpr int TILE_BYTES = TILE_ROWS * 128;
  static_assert(HP == 1 || HP * BS == TILE_ROWS, "packed heads fill one stage");
  static constexpr int NS = 8;
  static constexpr int NW = 4;
  static constexpr int min_ctas(int nt) { return nt == 1 ? 3 : 2; }  // two n-tiles: no spill at 2
  static constexpr int ZERO_CHUNKS_PER_ROW = 8;

  // K and V of the cache block at pool row `row` into block slot u of a stage
  __device__ static void issue(uint8_t* sk, uint8_t* sv, const CUtensorMap* mk,
                               const CUtensorMap* mv, int row, int u, uint64_t* bar,
                               uint64_t pol) {
    tma_load_2d(sk + u * BOX_BYTES, mk, 0, row, bar, pol);
    tma_load_2d(sv + u * BOX_BYTES, mv, 0, row, bar, pol);
  }
  __device__ static uint8_t* zero_chunk(uint8_t* v, int r, int idx) {
    return v + r * 128 + idx * 16;
  }
  // four E4M3 codes (one 32-bit word) -> two f16x2 words (bytes 0-1, 2-3)
  __device__ static void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
  }
  __device__ static uint32_t f16_pair(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  template <int NT>
  __device__ static void load_q(uint32_t (&qf)[D / 16][NT][2], const T* qbase, int G,
                                int lane) {
    const int c4 = lane & 3, r4 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + r4;
#pragma unroll
      for (int kt = 0; kt < D / 16; ++kt) {
        uint32_t b0 = 0, b1 = 0;
        if (g < G) {
          const T* row = qbase + (size_t)g * D + 32 * c4 + 4 * kt;
          b0 = f16_pair(float(row[0]), float(row[1]));
          b1 = f16_pair(float(row[2]), float(row[3]));
        }
        qf[kt][nt][0] = b0;
        qf[kt][nt][1] = b1;
      }
    }
  }
  // Tile reads are volatile shared loads: kept in program order they
  // measured faster here than compiler-scheduled loads.
  template <typename V>
  __device__ static V lds(const uint8_t* tile, int row, int col);
  template <int NT>
  __device__ static void qk(float (&sacc)[NT][4], const uint8_t* sk, int mt,
                            const uint32_t (&qf)[D / 16][NT][2], int lane) {
    const int c4 = lane & 3, r4 = lane >> 2;
    const int r_lo = mt * 16 + row_lo(r4), r_hi = r_lo + HI_STEP;
    uint4 lo[2], hi[2];  // bytes [32c, 32c+32) of rows r_lo, r_hi
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lo[h] = lds<uint4>(sk, r_lo, 32 * c4 + 16 * h);
      hi[h] = lds<uint4>(sk, r_hi, 32 * c4 + 16 * h);
    }
    float acc2[NT][4];  // odd k-steps accumulate separately (two shorter MMA chains)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc2[nt][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < D / 16; ++kt) {
      const uint4& L = lo[kt >> 2];
      const uint4& H = hi[kt >> 2];
      const uint32_t wl = (kt & 3) == 0 ? L.x : (kt & 3) == 1 ? L.y : (kt & 3) == 2 ? L.z : L.w;
      const uint32_t wh = (kt & 3) == 0 ? H.x : (kt & 3) == 1 ? H.y : (kt & 3) == 2 ? H.z : H.w;
      uint32_t a[4];
      e4m3x4_to_f16x2x2(wl, a[0], a[2]);
      e4m3x4_to_f16x2x2(wh, a[1], a[3]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        MmaOp<MmaT>::run((kt & 1) ? acc2[nt] : sacc[nt], a, qf[kt][nt][0], qf[kt][nt][1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] += acc2[nt][e];
  }
  // O^T += V^T P^T over a 16-token sub-tile.  ldmatrix .m16n16 .trans .b8
  // hands lane (g = lane / 4, c = lane % 4) the bytes of head dims 16 dt + g
  // and 16 dt + g + 8 for tokens 4c .. 4c + 3 — once converted, the A
  // fragment of m-tile dt with the sub-tile's tokens in the order row_lo
  // gives the S^T rows, so P^T (movmatrix of S^T) pairs with it as is.  One
  // .x2 load covers two m-tiles (lanes 0-15 address the token rows of the
  // first, 16-31 of the second).
  template <int NT>
  __device__ static void pv(float (&o)[D / 16][NT][4], const uint8_t* sv, int mt,
                            const uint32_t (&pb)[NT][2], int lane) {
    const uint32_t base = smem_u32(sv);
    const int row = mt * 16 + (lane & 15);
#pragma unroll
    for (int dt = 0; dt < D / 16; dt += 2) {
      const uint32_t addr = sw128(base, row, 16 * (dt + (lane >> 4)));
      uint32_t r[4];
      asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
                   : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                   : "r"(addr));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[4];
        e4m3x4_to_f16x2x2(r[2 * h], a[0], a[2]);      // head dim 16 (dt + h) + g
        e4m3x4_to_f16x2x2(r[2 * h + 1], a[1], a[3]);  // head dim 16 (dt + h) + g + 8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) MmaOp<MmaT>::run(o[dt + h][nt], a, pb[nt][0], pb[nt][1]);
      }
    }
  }
  __device__ static int out_d(int dt, int e, int r4) { return dt * 16 + r4 + (e >> 1) * 8; }
  // S^T accumulator rows r4 and r4 + 8 of a 16-row sub-tile hold tokens
  // row_lo(r4) and row_lo(r4) + HI_STEP of the sub-tile: 0 1 4 5 8 9 12 13
  // and 2 3 6 7 10 11 14 15 (qk loads K's rows in that order), the token
  // order of pv's fragments
  __device__ static int row_lo(int r4) { return 4 * (r4 >> 1) + (r4 & 1); }
  static constexpr int HI_STEP = 2;
};

template <typename T, int BS, int HP_>
template <typename V>
__device__ V E4m3Tiles<T, BS, HP_>::lds(const uint8_t* tile, int row, int col) {
  const uint32_t a = sw128(smem_u32(tile), row, col);
  if constexpr (sizeof(V) == 16) {
    V v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
  } else {
    V v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
  }
}

// --------------------------------------------------------------- kernel
template <class Tiles, int BS, int NT>
struct DecodeShape {
  static constexpr int D = Tiles::D;
  static constexpr int NW = Tiles::NW;              // consumer warps
  static constexpr int THREADS = (NW + 1) * 32;     // + producer warp
  static constexpr int TILE_BYTES = Tiles::TILE_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;   // K and V tiles of a stage
  static constexpr int HP = Tiles::HP;                  // KV heads per stage
  static constexpr int ROWS = Tiles::TILE_ROWS;         // tile rows per stage
  static constexpr int TT = ROWS / HP;                  // tokens per stage
  static constexpr int SB = TT / BS;                    // cache blocks per stage
  static constexpr int BLOCK_BYTES = STAGE_BYTES / SB;  // K + V bytes of one cache block
  static constexpr int NS = Tiles::NS;              // ring depth
  static constexpr int RING_BYTES = NS * STAGE_BYTES;
  static constexpr int MERGE_BYTES = NW * (NT * 8) * (D + 2) * 4;
  static constexpr int BODY_BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
  static constexpr int SMEM_BYTES = 1024 + BODY_BYTES + 2 * NS * 8 + 16;  // + abort word
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(BS == 16 || BS == 32, "block_size");
  // Consumer warp w takes ring positions w, w + NW, ... and waits on a
  // stage's full barrier by the parity of the fill it wants; with NS a
  // multiple of NW every stage is always consumed by the same warp, so no
  // warp can wait on a stage two fills ahead (where that parity test would
  // pass on an older phase).
  static_assert(NS % NW == 0, "ring depth vs consumer warps");
  static_assert(TT % BS == 0 && 32 % SB == 0 && ROWS % 16 == 0, "stage vs cache block");
  static_assert(HP == 1 || SB == 1, "a stage packs heads or blocks, not both");
};

// Length a work item attends over and its partition count.  A length beyond
// the table or beyond the launch's partitions (max_seq_len) is a caller error:
// it is flagged (by the item with flag_errors set) and clamped to what fits.
template <int BS>
__device__ __forceinline__ int decode_len(const DecodeParams& p, int s, bool flag_errors) {
  int L = p.seq_lens[s] + p.len_add;
  const int L_cap = min(p.max_blocks_per_seq, p.max_parts * p.part_blocks) * BS;
  if (L > L_cap) {
    if (flag_errors) record_error(PA_DEVERR_SEQ_RANGE);
    L = L_cap;
  }
  return L < 0 ? 0 : L;
}

__device__ __forceinline__ int decode_parts(int nblk_seq, int part_blocks) {
  return nblk_seq == 0 ? 1 : (nblk_seq + part_blocks - 1) / part_blocks;
}

// Producer side of one item: issue its nblk cache blocks (logical blocks
// blk0 .. blk0 + nblk - 1 of the block-table row `table`), SB per ring stage
// (the last stage of an item may hold fewer), into ring positions g0, g0 + 1,
// ... (position i uses stage i % NS and is that stage's (i / NS)-th fill).
// Block ids are fetched once, coalesced; entries past nblk are never read.
// Lane 0 waits, arms and loads; it returns (on lane 0) the first ring position
// not armed, `g0` plus the item's stages unless a wait gave up (`alive`
// false on lane 0), after which nothing more is armed or loaded.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ int produce_item(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                            const DecodeParams& p, uint8_t* ring,
                                            uint64_t* full_bar, uint64_t* empty_bar,
                                            const int32_t* table, int kvh, int blk0, int nblk,
                                            int g0, int lane, uint64_t policy, bool& alive,
                                            volatile int* abort) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  constexpr int NS = Shape::NS, SB = Shape::SB;
  const int32_t* bt = table + blk0;
  int armed = g0;
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
    for (int j = 0; j < cnt; j += SB) {
      int ph[SB];
#pragma unroll
      for (int u = 0; u < SB; ++u) ph[u] = __shfl_sync(0xffffffffu, phys, (j + u) & 31);
      if (lane == 0) {
        const int nb = min(SB, cnt - j);  // blocks in this stage
        const int i = g0 + (base + j) / SB, st = i % NS;
        if (i >= NS && alive) alive = mbar_wait(&empty_bar[st], ((i / NS) - 1) & 1, abort);
        if (alive) {
          mbar_arrive_expect_tx(&full_bar[st], nb * Shape::BLOCK_BYTES);
          uint8_t* sk = ring + st * Shape::STAGE_BYTES;
#pragma unroll
          for (int u = 0; u < SB; ++u)
            if (u < nb)
              Tiles::issue(sk, sk + Shape::TILE_BYTES, tm_k, tm_v,
                           (ph[u] * p.num_kv_heads + kvh * Shape::HP) * BS, u, &full_bar[st],
                           policy);
          armed = i + 1;
        }
      }
    }
  }
  return armed;
}

// Online softmax of one consumer warp over one ring stage (TT tokens of HP
// KV heads) whose first slot is logical position tok_blk: S^T = K Q^T,
// running max and sum, O^T += V^T P^T, on mma.sync with fp32 accumulation.
// Positions >= L (the end of the item's tokens) are masked and their V rows
// zeroed.  With HP > 1, tile rows [h*TT, (h+1)*TT) hold head h of the pack
// and only query columns [h*G, (h+1)*G) see them.
// Running max of the online softmax, per query column (the 8 lanes with the
// same lane % 4 hold a column's 16 rows): raised only when a sub-tile's column
// max exceeds it by more than 8 (log2 units), so P <= 2^8 stays in 16-bit
// range and O is rescaled rarely (the stale max cancels in O / l).
// running_max_may_rise: one warp vote on whether any lane holds a score above
// its column's m_run + 8 — when none does, no column max can exceed it either,
// and the per-column shuffle reductions are skipped (the common case).
template <int NT>
__device__ __forceinline__ bool running_max_may_rise(const float (&sl)[NT][2],
                                                     const float (&sh)[NT][2],
                                                     const float (&m_run)[NT][2]) {
  bool above = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) above |= fmaxf(sl[nt][j], sh[nt][j]) > m_run[nt][j] + 8.f;
  return __any_sync(0xffffffffu, above);
}
// The column maxima (3 shuffles each) and the raise; alpha = 2^(old - new)
// for raised columns (0 when the old max was -inf).  Returns this lane's
// "some column rose".
template <int NT>
__device__ __forceinline__ bool raise_running_max(const float (&sl)[NT][2],
                                                  const float (&sh)[NT][2], float (&m_run)[NT][2],
                                                  float (&alpha)[NT][2]) {
  bool raise = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float mx = fmaxf(sl[nt][j], sh[nt][j]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (mx > m_run[nt][j] + 8.f) {
        alpha[nt][j] = ex2_approx(m_run[nt][j] - mx);
        m_run[nt][j] = mx;
        raise = true;
      }
    }
  return raise;
}

// consume_block for a stage of two packed KV heads (rows 0-15: head 0's
// tokens, rows 16-31: head 1's, the same 16 positions; t_lo is the position
// of this lane's S^T accumulator row, Tiles::row_lo): query
// column g belongs to head g / G (g >= 2G: padding), so each column uses the
// scores of one sub-tile only and one online-softmax pass (one max
// reduction, four exponentials per lane) serves both; P of each sub-tile keeps
// only its head's columns.  The per-column arithmetic is that of two
// separate passes (the other pass only adds zeros), so the result is the same
// bit for bit.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void consume_packed_pair(
    float (&o)[Tiles::D / 16][NT][4], float (&m_run)[NT][2], float (&l_run)[NT][2],
    const uint32_t (&qf)[Tiles::D / 16][NT][2], const uint8_t* sk, const uint8_t* sv, int t_lo,
    int L, float scale_log2, int lane, int G) {
  using MmaT = typename Tiles::MmaT;
  constexpr int D = Tiles::D;
  const int c4 = lane & 3;
  float sacc[2][NT][4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[hh][nt][e] = 0.f;
  Tiles::template qk<NT>(sacc[0], sk, 0, qf, lane);
  Tiles::template qk<NT>(sacc[1], sk, 1, qf, lane);
  const bool ok_lo = t_lo < L, ok_hi = t_lo + Tiles::HI_STEP < L;
  int head[NT][2];
  float sl[NT][2], sh[NT][2], alpha[NT][2];
  bool raise = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hc = (nt * 8 + 2 * c4 + j) / G;
      head[nt][j] = hc;
      const float lo = hc == 0 ? sacc[0][nt][j] : sacc[1][nt][j];
      const float hi = hc == 0 ? sacc[0][nt][j + 2] : sacc[1][nt][j + 2];
      sl[nt][j] = ok_lo && hc < 2 ? lo * scale_log2 : -INFINITY;
      sh[nt][j] = ok_hi && hc < 2 ? hi * scale_log2 : -INFINITY;
      alpha[nt][j] = 1.f;
    }
  if (running_max_may_rise<NT>(sl, sh, m_run))
    raise = raise_running_max<NT>(sl, sh, m_run, alpha);
  if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        l_run[nt][j] *= alpha[nt][j];
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
          o[dt][nt][j] *= alpha[nt][j];
          o[dt][nt][j + 2] *= alpha[nt][j];
        }
      }
  }
  uint32_t pb[2][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float pv[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float m_use = m_run[nt][j] == -INFINITY ? 0.f : m_run[nt][j];
      pv[j] = ex2_approx(sl[nt][j] - m_use);
      pv[j + 2] = ex2_approx(sh[nt][j] - m_use);
      l_run[nt][j] += pv[j] + pv[j + 2];
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const bool m0 = head[nt][0] == hh, m1 = head[nt][1] == hh;
      pb[hh][nt][0] = movmatrix_trans(MmaOp<MmaT>::pack(m0 ? pv[0] : 0.f, m1 ? pv[1] : 0.f));
      pb[hh][nt][1] = movmatrix_trans(MmaOp<MmaT>::pack(m0 ? pv[2] : 0.f, m1 ? pv[3] : 0.f));
    }
  }
  Tiles::template pv<NT>(o, sv, 0, pb[0], lane);
  Tiles::template pv<NT>(o, sv, 1, pb[1], lane);
}

template <class Tiles, int BS, int NT>
__device__ __forceinline__ void consume_block(float (&o)[Tiles::D / 16][NT][4],
                                              float (&m_run)[NT][2], float (&l_run)[NT][2],
                                              const uint32_t (&qf)[Tiles::D / 16][NT][2],
                                              uint8_t* sk, int tok_blk, int L, float scale_log2,
                                              int lane, int G = 0) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  using MmaT = typename Tiles::MmaT;
  constexpr int D = Shape::D, TT = Shape::TT, HP = Shape::HP;
  const int r4 = lane >> 2, c4 = lane & 3;
  uint8_t* sv = sk + Shape::TILE_BYTES;
  const int valid = min(TT, L - tok_blk);
  if (valid < TT) {
    // Slots past the sequence end may hold anything (NaN included); zero
    // their V rows so that 0-weight x garbage cannot poison the PV product.
    constexpr int CPR = Tiles::ZERO_CHUNKS_PER_ROW;
    const int per_head = (TT - valid) * CPR;
    for (int idx = lane; idx < HP * per_head; idx += 32) {
      const int h = idx / per_head, k = idx % per_head;
      *reinterpret_cast<uint4*>(Tiles::zero_chunk(sv, h * TT + valid + k / CPR, k % CPR)) =
          make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
  }
  if constexpr (HP == 2) {
    consume_packed_pair<Tiles, BS, NT>(o, m_run, l_run, qf, sk, sv, tok_blk + Tiles::row_lo(r4),
                                       L, scale_log2, lane, G);
  } else {
#pragma unroll
    for (int mt = 0; mt < Shape::ROWS / 16; ++mt) {
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
      Tiles::template qk<NT>(sacc, sk, mt, qf, lane);
      // online softmax over this sub-tile's 16 rows (tokens of one head)
      const int t_lo = tok_blk + (mt * 16) % TT + Tiles::row_lo(r4);
      bool ok_lo = t_lo < L, ok_hi = t_lo + Tiles::HI_STEP < L;
      bool col_ok[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          col_ok[nt][j] = HP == 1 || (nt * 8 + 2 * c4 + j) / G == (mt * 16) / TT;
      // running max: see running_max_may_rise / raise_running_max
      uint32_t pb[NT][2];
      float sl[NT][2], sh[NT][2], alpha[NT][2];
      bool raise = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          sl[nt][j] = ok_lo && col_ok[nt][j] ? sacc[nt][j] * scale_log2 : -INFINITY;
          sh[nt][j] = ok_hi && col_ok[nt][j] ? sacc[nt][j + 2] * scale_log2 : -INFINITY;
          alpha[nt][j] = 1.f;
        }
      if (running_max_may_rise<NT>(sl, sh, m_run))
        raise = raise_running_max<NT>(sl, sh, m_run, alpha);
      if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            l_run[nt][j] *= alpha[nt][j];
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
              o[dt][nt][j] *= alpha[nt][j];
              o[dt][nt][j + 2] *= alpha[nt][j];
            }
          }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float pv[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float m_use = m_run[nt][j] == -INFINITY ? 0.f : m_run[nt][j];
          pv[j] = ex2_approx(sl[nt][j] - m_use);
          pv[j + 2] = ex2_approx(sh[nt][j] - m_use);
          l_run[nt][j] += pv[j] + pv[j + 2];
        }
        // accumulator rows t / t+8, cols (g, g+1) -> B-operand layout of P^T
        pb[nt][0] = movmatrix_trans(MmaOp<MmaT>::pack(pv[0], pv[1]));
        pb[nt][1] = movmatrix_trans(MmaOp<MmaT>::pack(pv[2], pv[3]));
      }
      Tiles::template pv<NT>(o, sv, mt, pb, lane);
    }
  }
  if (valid < TT) fence_proxy_async_smem();  // our zero stores precede the next TMA write
}

// Merge the NW consumer warps' states of one item in shared memory `mg`
// ([NW][8 NT][D + 2] floats) in warp order, then write the output row (one
// partition) or the partition's (m, l, acc) to the workspace.  Query column
// g (g < cols) belongs to sequence s + g / G and query head kvh * G + g % G
// (G = the item's query heads per sequence); single_of(seq) says whether that
// sequence has one partition.  Opens with a barrier of the consumer warps, so
// `mg` may alias the item's ring or the previous item's merge area.
template <class Tiles, int BS, int NT, class SingleOf>
__device__ __forceinline__ void merge_item(float* mg, float (&o)[Tiles::D / 16][NT][4],
                                           float (&m_run)[NT][2], float (&l_run)[NT][2],
                                           const DecodeParams& p, int s, int kvh, int part,
                                           int cols, SingleOf single_of, int ctid,
                                           uint32_t bar_consumers) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  constexpr int D = Shape::D, NW = Shape::NW;
  constexpr int GP = NT * 8;  // padded heads per item
  const int warp = ctid >> 5, lane = ctid & 31;
  const int c4 = lane & 3, r4 = lane >> 2;
  const int G = p.group * Shape::HP;  // query heads of the item (kvh is a pack index)
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
  named_barrier(bar_consumers, NW * 32);  // every consumer is done with `mg`'s old contents
  constexpr int RS = D + 2;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int g = nt * 8 + 2 * c4 + (e & 1);
        mg[(warp * GP + g) * RS + Tiles::out_d(dt, e, r4)] = o[dt][nt][e];
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
  named_barrier(bar_consumers, NW * 32);
  for (int idx = ctid; idx < cols * D; idx += NW * 32) {
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
    num *= p.v_scale;
    const int sq = s + g / G;
    const int h = kvh * G + g % G;  // == (kvh * HP) * group + g for one sequence
    if (single_of(sq)) {
      const float v = den > 0.f ? num / den : 0.f;
      reinterpret_cast<T*>(p.out)[((size_t)sq * p.num_q_heads + h) * D + d] = T(v);
    } else {
      const size_t row = ((size_t)sq * p.num_q_heads + h) * p.max_parts + part;
      p.ws_acc[row * D + d] = num;
      if (d == 0) {
        p.ws_ml[row * 2] = M;
        p.ws_ml[row * 2 + 1] = den;
      }
    }
  }
}

template <class Tiles, int NT>
__device__ __forceinline__ void reset_state(float (&o)[Tiles::D / 16][NT][4],
                                            float (&m_run)[NT][2], float (&l_run)[NT][2]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int dt = 0; dt < Tiles::D / 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[dt][nt][e] = 0.f;
  }
}

// Fused append, by the producer warp of the item that holds logical position
// `pos` (the sequence's new token): write the token's K and V rows of the
// item's KV heads (Tiles::HP of them, from pack index kvp) into its slot
// (block_tables[s][pos / BS], offset pos % BS), 16 bytes per lane — bit
// copies for fp16 / bf16 caches, E4M3 codes of value / scale (the rule of
// pa_reshape_and_cache_fp8) for FP8 caches — then order those writes before
// this CTA's TMA reads of the block.  An out-of-pool block id is flagged and
// not written.
template <class Tiles, int BS>
__device__ __forceinline__ void append_new_token(const DecodeParams& p, int s, int kvp, int pos,
                                                 int lane) {
  using T = typename Tiles::Elem;
  constexpr int D = Tiles::D, HP = Tiles::HP;
  constexpr int CB = Tiles::kHalfCache ? 2 : 1;  // cache bytes per element
  constexpr int CH = D * CB / 16;                // 16-byte chunks per cache row
  const int32_t blk = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + pos / BS);
  const bool ok = blk >= 0 && blk < p.num_blocks;
  if (ok) {
    for (int i = lane; i < 2 * HP * CH; i += 32) {
      const bool is_v = i >= HP * CH;
      const int r = is_v ? i - HP * CH : i;
      const int h = kvp * HP + r / CH, c = r % CH;
      const size_t row = ((size_t)blk * p.num_kv_heads + h) * BS + pos % BS;
      const T* src = reinterpret_cast<const T*>(is_v ? p.new_value : p.new_key) +
                     ((size_t)s * p.num_kv_heads + h) * D + c * (16 / CB);
      uint4 v;
      if constexpr (Tiles::kHalfCache)
        v = __ldg(reinterpret_cast<const uint4*>(src));
      else
        v = quantize16_e4m3<T>(src, is_v ? p.v_scale : p.k_scale);
      reinterpret_cast<uint4*>(is_v ? p.value_cache : p.key_cache)[row * CH + c] = v;
    }
  } else if (lane == 0) {
    record_error(PA_DEVERR_BLOCK_RANGE);
  }
  if (lane == 0 && kvp == 0 && p.slot_out != nullptr)
    p.slot_out[s] = ok ? (int64_t)blk * BS + pos % BS : -1;
  fence_proxy_async_global();
  __syncwarp();
}

// Ring protocol of one work item.  The producer warp issues the first NS ring
// positions (item_ring_fill); after that the consumer warp that finishes
// position i issues position i + NS into the same stage itself (NS is a
// multiple of NW, so that position is its own), so a stage is refilled the
// moment it is free, never behind another warp's slower stage.
// last_fill[st] (shared) is the last position issued on stage st, for the
// drain after an abort (item_ring_drain); the empty barriers are not used.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void item_ring_init(uint64_t* full_bar, int* last_fill, int nstages) {
  constexpr int NS = DecodeShape<Tiles, BS, NT>::NS;
  for (int i = 0; i < NS; ++i) {
    mbar_init(&full_bar[i], 1);
    last_fill[i] = i < nstages ? i : -1;
  }
}
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void item_ring_fill(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                               const DecodeParams& p, uint8_t* smem,
                                               uint64_t* full_bar, uint64_t* empty_bar,
                                               const int32_t* table, int kvh, int blk0, int nblk,
                                               int lane, uint64_t policy, volatile int* abort) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  bool alive = true;  // positions < NS wait for nothing: all of them are issued
  produce_item<Tiles, BS, NT>(tm_k, tm_v, p, smem, full_bar, empty_bar, table, kvh, blk0,
                              min(nblk, Shape::NS * Shape::SB), 0, lane, policy, alive, abort);
}
// After an abort (one thread): let every load still in flight land.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void item_ring_drain(uint64_t* full_bar, const int* last_fill) {
  constexpr int NS = DecodeShape<Tiles, BS, NT>::NS;
  for (int st = 0; st < NS; ++st)
    if (last_fill[st] >= 0) mbar_drain(&full_bar[st], (last_fill[st] / NS) & 1);
}

// Consumer side of one item (blocks blk0 .. blk0 + nblk - 1 of the table row
// `bt`, which starts at block blk0): consume_block over the warp's ring
// positions, each followed by the refill of its stage.  The warp's refill
// block ids sit in a register window: lane l holds the blocks of the warp's
// (kw + l)-th position, fetched 32 positions at a time.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void consume_item(
    float (&o)[Tiles::D / 16][NT][4], float (&m_run)[NT][2], float (&l_run)[NT][2],
    const uint32_t (&qf)[Tiles::D / 16][NT][2], const CUtensorMap* tm_k, const CUtensorMap* tm_v,
    const DecodeParams& p, uint8_t* smem, uint64_t* full_bar, int* last_fill,
    const int32_t* bt, int kvh, int blk0, int nblk, int L_end, int G, uint64_t policy, int warp,
    int lane, volatile int* abort) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  constexpr int NW = Shape::NW, NS = Shape::NS, SB = Shape::SB;
  const int nstages = (nblk + SB - 1) / SB;
  int ids[SB];
  int kw = -32;
  bool alive = true;
  for (int i = warp; i < nstages; i += NW) {
    const int st = i % NS;
    // after a wait gave up the warp still runs through its (garbage) stages,
    // every lane alike, so the .aligned loads and MMAs stay converged
    if (alive) alive = mbar_wait(&full_bar[st], (i / NS) & 1, abort);
    consume_block<Tiles, BS, NT>(o, m_run, l_run, qf, smem + st * Shape::STAGE_BYTES,
                                 (blk0 + i * SB) * BS, L_end, p.scale_log2, lane, G);
    __syncwarp();
    const int nxt = i + NS;  // the next fill of stage st (warp-uniform test)
    if (nxt < nstages) {
      const int k = (nxt - warp) / NW;
      if (k >= kw + 32) {
        kw = k;
#pragma unroll
        for (int u = 0; u < SB; ++u) {
          const int b = (warp + NW * (k + lane)) * SB + u;
          int id = 0;
          if (b < nblk) {
            id = __ldg(bt + b);
            if (id < 0 || id >= p.num_blocks) {
              record_error(PA_DEVERR_BLOCK_RANGE);
              id = 0;
            }
          }
          ids[u] = id;
        }
      }
      int ph[SB];
#pragma unroll
      for (int u = 0; u < SB; ++u) ph[u] = __shfl_sync(0xffffffffu, ids[u], k - kw);
      if (lane == 0 && alive) {
        // this warp's reads of the stage are done (__syncwarp above); order
        // them before the async-proxy writes that refill it
        fence_proxy_async_smem();
        const int nb = min(SB, nblk - nxt * SB);
        mbar_arrive_expect_tx(&full_bar[st], nb * Shape::BLOCK_BYTES);
        uint8_t* sk = smem + st * Shape::STAGE_BYTES;
#pragma unroll
        for (int u = 0; u < SB; ++u)
          if (u < nb)
            Tiles::issue(sk, sk + Shape::TILE_BYTES, tm_k, tm_v,
                         (ph[u] * p.num_kv_heads + kvh * Shape::HP) * BS, u, &full_bar[st],
                         policy);
        last_fill[st] = nxt;
      }
    }
  }
}

// One work item (split-KV partition `part` of KV head `kvh` of sequence `s`)
// run by THREADS consecutive threads (`tid` 0 .. THREADS-1) that own the
// 1024-byte aligned shared memory at `smem` (SMEM_BYTES - 1024 bytes).  They
// synchronise among themselves only, on named barriers `bar_all` (all
// THREADS) and `bar_consumers` (the NW consumer warps).  A wait that gives up
// ends the item: the producer stops loading, the consumers skip the rest, and
// the producer drains its loads in flight before the threads leave.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void decode_item(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                            const DecodeParams& p, uint8_t* smem, int part,
                                            int kvh, int s, int tid, uint32_t bar_all,
                                            uint32_t bar_consumers) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  constexpr int D = Shape::D, NW = Shape::NW, NS = Shape::NS;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Shape::BODY_BYTES);
  uint64_t* empty_bar = full_bar + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty_bar + NS);
  const int warp = tid >> 5, lane = tid & 31;

  const int L = decode_len<BS>(p, s, tid == 0 && part == p.part_base && kvh == 0);
  const int nblk_seq = (L + BS - 1) / BS;
  const int nparts = decode_parts(nblk_seq, p.part_blocks);
  if (part >= nparts) return;
  const int blk0 = part * p.part_blocks;
  const int nblk = min(p.part_blocks, nblk_seq - blk0);  // 0 only when L == 0

  // ring protocol: item_ring_init; the empty barriers' memory holds last_fill
  const int nstages = (nblk + Shape::SB - 1) / Shape::SB;
  int* last_fill = reinterpret_cast<int*>(empty_bar);
  if (tid == 0) {
    item_ring_init<Tiles, BS, NT>(full_bar, last_fill, nstages);
    *abort = 0;
    fence_barrier_init();
  }
  named_barrier(bar_all, Shape::THREADS);

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(tm_k);
      tma_prefetch_desc(tm_v);
    }
    // fused append: the new token is the last position; skipped when the
    // length was clamped (flagged by decode_len)
    if (p.new_key != nullptr && part == nparts - 1) {
      if (L >= 1 && p.seq_lens[s] + p.len_add == L)
        append_new_token<Tiles, BS>(p, s, kvh, L - 1, lane);
      else if (lane == 0 && kvh == 0 && p.slot_out != nullptr)
        p.slot_out[s] = -1;
    }
    item_ring_fill<Tiles, BS, NT>(tm_k, tm_v, p, smem, full_bar, empty_bar,
                                  p.block_tables + (size_t)s * p.max_blocks_per_seq, kvh, blk0,
                                  nblk, lane, l2_policy_evict_first(), abort);
    named_barrier(bar_all, Shape::THREADS);  // the consumers are done
    if (*abort && lane == 0) item_ring_drain<Tiles, BS, NT>(full_bar, last_fill);
    return;
  }

  // -------------------------------------------------------------- consumers
  uint32_t qf[D / 16][NT][2];  // Q^T as the B operand
  const int G_item = p.group * Shape::HP;  // query heads of this item
  Tiles::template load_q<NT>(
      qf, reinterpret_cast<const T*>(p.query) +
              ((size_t)s * p.num_q_heads + (size_t)kvh * G_item) * D,
      G_item, lane);
  float m_run[NT][2], l_run[NT][2];
  float o[D / 16][NT][4];
  reset_state<Tiles, NT>(o, m_run, l_run);
  // a stage may reach past the item's last block (into the next partition)
  const int L_end = min(L, (blk0 + nblk) * BS);
  consume_item<Tiles, BS, NT>(o, m_run, l_run, qf, tm_k, tm_v, p, smem, full_bar, last_fill,
                              p.block_tables + (size_t)s * p.max_blocks_per_seq + blk0, kvh, blk0,
                              nblk, L_end, p.group, l2_policy_evict_first(), warp, lane, abort);
  // the merge area aliases the ring: merge_item's opening barrier waits for
  // every consumer to finish reading it (after an abort a late load may still
  // land there; the output is garbage then, and the error word says so)
  merge_item<Tiles, BS, NT>(reinterpret_cast<float*>(smem), o, m_run, l_run, p, s, kvh, part,
                            G_item, [&](int) { return nparts == 1; }, tid, bar_consumers);
  named_barrier(bar_all, Shape::THREADS);  // lets the producer see the final abort word
}

template <class Tiles, int BS, int NT>
__global__ void __launch_bounds__(DecodeShape<Tiles, BS, NT>::THREADS, Tiles::min_ctas(NT))
    decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // the split-KV combine that follows may be launched (it waits for this grid)
  griddep_launch_dependents();
  decode_item<Tiles, BS, NT>(&tm_k, &tm_v, p, smem, p.part_base + blockIdx.x, blockIdx.y,
                             blockIdx.z, threadIdx.x, 0, 1);
  // launched to overlap a shared-prefix pass: finish only after it (so the
  // combine, which waits for this grid, sees its partials)
  griddep_wait();
}

// Shared-prefix partitions (pa_decode_shared_prefix).  Every sequence of the
// batch starts with the same physical blocks, prefix_blocks; partition `part`
// (logical blocks part * part_blocks .. (part + 1) * part_blocks - 1, all of
// them shared) is the same K/V for every sequence.  One CTA per (partition,
// KV head, group of seq_group sequences) streams those tiles once and applies
// them to the query heads of all the group's sequences, side by side in the
// MMA's query columns (NT = 2: 16 columns).  Each column's arithmetic — the
// score and P fragments, the per-warp online softmax, the merge over warps in
// warp order — is exactly what pa_decode's CTA for that sequence does on the
// same partition, so the partials (or, for a one-partition sequence, the
// output row) are bit-identical to pa_decode's.
template <class Tiles, int BS>
__global__ void __launch_bounds__(DecodeShape<Tiles, BS, 2>::THREADS, Tiles::min_ctas(2))
    prefix_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, DecodeParams p) {
  constexpr int NT = 2;
  using Shape = DecodeShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  constexpr int D = Shape::D, NW = Shape::NW, NS = Shape::NS;
  static_assert(Shape::HP == 1, "fp16 / bf16 caches only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Shape::BODY_BYTES);
  uint64_t* empty_bar = full_bar + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty_bar + NS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int part = blockIdx.x, kvh = blockIdx.y;
  const int s0 = blockIdx.z * p.seq_group;
  const int nseq = min(p.seq_group, p.num_seqs - s0);
  const int G = p.group;
  const int blk0 = part * p.part_blocks, nblk = p.part_blocks;
  const int L_end = (blk0 + nblk) * BS;  // every token of the partition is valid

  const int nstages = (nblk + Shape::SB - 1) / Shape::SB;
  int* last_fill = reinterpret_cast<int*>(empty_bar);  // ring protocol: item_ring_init
  if (tid == 0) {
    item_ring_init<Tiles, BS, NT>(full_bar, last_fill, nstages);
    *abort = 0;
    fence_barrier_init();
    // every sequence must hold the whole shared partition
    if (kvh == 0)
      for (int j = 0; j < nseq; ++j)
        if (decode_len<BS>(p, s0 + j, false) < L_end) record_error(PA_DEVERR_SEQ_RANGE);
  }
  named_barrier(0, Shape::THREADS);
  // the rest of the sequences' partitions (decode_kernel) may start now: they
  // write other partitions and wait for this grid before they finish
  griddep_launch_dependents();

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    // the shared tiles are read by every group's CTA: keep them in L2
    item_ring_fill<Tiles, BS, NT>(&tm_k, &tm_v, p, smem, full_bar, empty_bar, p.prefix_blocks,
                                  kvh, blk0, nblk, lane, l2_policy_evict_last(), abort);
    named_barrier(0, Shape::THREADS);  // the consumers are done
    if (*abort && lane == 0) item_ring_drain<Tiles, BS, NT>(full_bar, last_fill);
    return;
  }

  // -------------------------------------------------------------- consumers
  uint32_t qf[D / 16][NT][2];
  const int cols = nseq * G;
  Tiles::template load_q_cols<NT>(
      qf,
      [&](int g) -> const T* {
        if (g >= cols) return nullptr;
        return reinterpret_cast<const T*>(p.query) +
               ((size_t)(s0 + g / G) * p.num_q_heads + (size_t)kvh * G + g % G) * D;
      },
      lane);
  float m_run[NT][2], l_run[NT][2];
  float o[D / 16][NT][4];
  reset_state<Tiles, NT>(o, m_run, l_run);
  consume_item<Tiles, BS, NT>(o, m_run, l_run, qf, &tm_k, &tm_v, p, smem, full_bar, last_fill,
                              p.prefix_blocks + blk0, kvh, blk0, nblk, L_end, G,
                              l2_policy_evict_last(), warp, lane, abort);
  merge_item<Tiles, BS, NT>(
      reinterpret_cast<float*>(smem), o, m_run, l_run, p, s0, kvh, part, cols,
      [&](int sq) {
        return decode_parts((decode_len<BS>(p, sq, false) + BS - 1) / BS, p.part_blocks) == 1;
      },
      tid, 1);
  named_barrier(0, Shape::THREADS);  // lets the producer see the final abort word
}

// Log-sum-exp combine of split-KV partitions, in partition order.  One warp
// per (sequence, query head), REDUCE_WARPS warps per CTA, so the whole grid
// is one wave of short-lived warps; lane l owns D / 32 consecutive head-dim
// elements (one vector load per partition).  Per element the arithmetic is
// M = max_q m_q, num = sum_q 2^(m_q - M) acc_q, den = sum_q 2^(m_q - M) l_q
// in partition order.  Sequences that fit one partition were finished by
// decode_kernel and are skipped.
constexpr int REDUCE_WARPS = 8;

template <typename T, int D>
__global__ void __launch_bounds__(REDUCE_WARPS * 32)
    decode_reduce_kernel(DecodeParams p, int block_size) {
  constexpr int VPL = D / 32;  // elements per lane: 4 (D = 128) or 2 (D = 64)
  griddep_wait();  // launched early: the partials are complete only after this
  const int lane = threadIdx.x & 31;
  const int unit = blockIdx.x * REDUCE_WARPS + (threadIdx.x >> 5);
  if (unit >= p.num_seqs * p.num_q_heads) return;
  const int s = unit / p.num_q_heads, h = unit % p.num_q_heads;
  int L = p.seq_lens[s] + p.len_add;
  L = max(0, min(L, min(p.max_blocks_per_seq, p.max_parts * p.part_blocks) * block_size));
  const int nblk = (L + block_size - 1) / block_size;
  const int nparts = nblk == 0 ? 1 : (nblk + p.part_blocks - 1) / p.part_blocks;
  if (nparts <= 1) return;
  const size_t row0 = ((size_t)s * p.num_q_heads + h) * p.max_parts;
  float M = -INFINITY;
#pragma unroll 4
  for (int q = 0; q < nparts; ++q) M = fmaxf(M, __ldg(p.ws_ml + (row0 + q) * 2));
  const float m_use = M == -INFINITY ? 0.f : M;
  float num[VPL], den = 0.f;
#pragma unroll
  for (int e = 0; e < VPL; ++e) num[e] = 0.f;
#pragma unroll 4
  for (int q = 0; q < nparts; ++q) {
    const float sc = exp2f(__ldg(p.ws_ml + (row0 + q) * 2) - m_use);
    const float* acc = p.ws_acc + (row0 + q) * D + lane * VPL;
    float a[VPL];
    if constexpr (VPL == 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(acc));
      a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
    } else {
      const float2 v = __ldg(reinterpret_cast<const float2*>(acc));
      a[0] = v.x; a[1] = v.y;
    }
#pragma unroll
    for (int e = 0; e < VPL; ++e) num[e] += sc * a[e];
    den += sc * __ldg(p.ws_ml + (row0 + q) * 2 + 1);
  }
  T* o = reinterpret_cast<T*>(p.out) + ((size_t)s * p.num_q_heads + h) * D + lane * VPL;
#pragma unroll
  for (int e = 0; e < VPL; ++e) o[e] = T(den > 0.f ? num[e] / den : 0.f);
}

}  // namespace pa
