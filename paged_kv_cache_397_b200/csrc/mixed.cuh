// mixed.cuh — one launch for a batch that mixes decode rows and prefill chunks.
//
// What it computes ("vLLM PagedAttention Deep Dive", "Mechanics of Chunked
// Prefill": the scheduler puts the ongoing decode tokens and a chunk of a long
// prompt into the same batch): every query row of the batch attends causally
// to its own sequence's paged K/V.  Sequence s has ctx_lens[s] tokens cached
// before this step and cu_q_lens[s+1] - cu_q_lens[s] query rows whose K/V are
// already in the cache; chunk row i sees positions 0 .. ctx_lens[s] + i.  A
// decode row is the one-row case: it sees ctx_lens[s] + 1 tokens.
//
// How (B200 design).  The first num_decode sequences are decode rows (one
// query each, at row s); the rest are prefill chunks.  One grid of CTAs (512
// threads with one query n-tile, 384 with two) covers both kinds of work:
//  * a prefill CTA runs one 256-row prefill tile on the tcgen05 tensor cores
//    (prefill_tile, the same code as pa_prefill_chunk);
//  * a decode CTA (at most one per SM) hosts persistent decode workers of 160
//    threads (a producer warp and four consumer warps, on their own named
//    barriers and shared memory).  A worker's producer takes split-KV work
//    items (partition, KV head, decode sequence) from an atomic queue in the
//    workspace and streams their (block, KV head) tiles through one TMA ring
//    without draining it between items; the consumers process each item
//    exactly as pa_decode's CTA does (same warp for each block, same merge
//    order), so the results are bit-identical to pa_decode.
// Launch order (MixedPlan): a leading share of the prefill tiles, decode CTAs
// for the other SMs, the remaining tiles, then the remaining decode CTAs.
// The hardware hands out clusters in order, so the tensor-bound tiles and the
// HBM-bound decode run side by side from the start; later tiles take the SMs
// the first ones free, the last decode CTAs take the SMs the tiles leave, and
// the queue keeps every worker busy until it is drained.  The grid runs as
// clusters of two CTAs, which share a TPC (the two SMs of a tcgen05 CTA
// pair), and both CTAs of a cluster do the same kind of work: on B200 a
// prefill tile whose TPC partner SM ran decode workers was measured at about
// half speed, so a TPC runs two prefill tiles or two decode CTAs, never one
// of each.  Decode items that span several partitions are combined
// afterwards by decode_reduce_kernel.
#pragma once

#include "decode.cuh"
#include "prefill.cuh"

namespace pa {

// Shared memory of one persistent decode worker: the TMA ring, a merge area
// of its own (so the producer can stream the next item while the consumers
// merge this one; two warps' partial O at a time plus every warp's (m, l)),
// ring and item-handoff mbarriers, the item slots, and the item the
// consumers are working on.
template <class Tiles, int BS, int NT>
struct WorkerShape {
  using Dc = DecodeShape<Tiles, BS, NT>;
  static constexpr int QD = 2;  // item slots between producer and consumers
  static constexpr int GP = NT * 8;
  static constexpr int MERGE_BYTES = (2 * GP * (Dc::D + 2) + Dc::NW * GP * 2) * 4;
  static constexpr int MERGE_OFF = Dc::RING_BYTES;
  static constexpr int BAR_OFF = MERGE_OFF + MERGE_BYTES;
  static constexpr int NBAR = 2 * Dc::NS + 2 * QD;
  static constexpr int ITEM_OFF = BAR_OFF + NBAR * 8;
  // item slots, the current item, the worker's abort word, the last ring
  // position filled on each stage
  static constexpr int BYTES = (ITEM_OFF + (QD + 2 + Dc::NS) * 4 + 1023) / 1024 * 1024;
};

// Merge of one item's four consumer-warp states for a decode worker, through
// a merge area half the size of merge_item's: every warp's (m, l) first, then
// the partial O of warps 0-1 and, after them, of warps 2-3.  Each output
// element is accumulated by the same thread in warp order w = 0, 1, 2, 3 with
// the same operations as merge_item, so the result is bit-identical to
// pa_decode's.
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void merge_item_two_pass(float* mg, float (&o)[Tiles::D / 16][NT][4],
                                                    float (&m_run)[NT][2], float (&l_run)[NT][2],
                                                    const DecodeParams& p, int s, int kvh,
                                                    int part, bool single, int ctid,
                                                    uint32_t bar_consumers) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  constexpr int D = Shape::D, NW = Shape::NW, GP = NT * 8, RS = D + 2;
  constexpr int KMAX = GP * D / (NW * 32);  // output elements per thread (at most)
  static_assert(NW == 4 && Shape::HP == 1, "four consumer warps, one KV head per item");
  float* ml = mg + 2 * GP * RS;  // [NW][GP][2]
  const int warp = ctid >> 5, lane = ctid & 31;
  const int c4 = lane & 3, r4 = lane >> 2;
  const int G = p.group;
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
  auto put_o = [&](int slot) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mg[(slot * GP + nt * 8 + 2 * c4 + (e & 1)) * RS + Tiles::out_d(dt, e, r4)] =
              o[dt][nt][e];
  };
  if (r4 == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int g = nt * 8 + 2 * c4 + j;
        ml[(warp * GP + g) * 2] = m_run[nt][j];
        ml[(warp * GP + g) * 2 + 1] = l_run[nt][j];
      }
  }
  if (warp < 2) put_o(warp);
  named_barrier(bar_consumers, NW * 32);
  float num[KMAX], den[KMAX];
  auto accumulate = [&](int w0) {
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      const int idx = ctid + k * NW * 32;
      if (idx >= G * D) continue;
      const int g = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, ml[(w * GP + g) * 2]);
      const float m_use = M == -INFINITY ? 0.f : M;
      if (w0 == 0) num[k] = den[k] = 0.f;
#pragma unroll
      for (int w = w0; w < w0 + 2; ++w) {
        const float sc = exp2f(ml[(w * GP + g) * 2] - m_use);
        num[k] += sc * mg[((w - w0) * GP + g) * RS + d];
        den[k] += sc * ml[(w * GP + g) * 2 + 1];
      }
      if (w0 == 2) {
        const float nv = num[k] * p.v_scale;
        const int h = kvh * G + g;
        if (single) {
          const float v = den[k] > 0.f ? nv / den[k] : 0.f;
          reinterpret_cast<T*>(p.out)[((size_t)s * p.num_q_heads + h) * D + d] = T(v);
        } else {
          const size_t row = ((size_t)s * p.num_q_heads + h) * p.max_parts + part;
          p.ws_acc[row * D + d] = nv;
          if (d == 0) {
            p.ws_ml[row * 2] = M;
            p.ws_ml[row * 2 + 1] = den[k];
          }
        }
      }
    }
  };
  accumulate(0);                          // warps 0 and 1
  named_barrier(bar_consumers, NW * 32);  // their partial O has been read
  if (warp >= 2) put_o(warp - 2);
  named_barrier(bar_consumers, NW * 32);
  accumulate(2);                          // warps 2 and 3, then the output
}

// Work item i of the decode queue, in partition-major order: partition 0 of
// every (sequence, KV head), then partition 1, and so on, so the last items
// handed out are the late partitions of the longest sequences, most of them
// shorter than a partition, and the workers finish close together.
__device__ __forceinline__ void worker_item(const DecodeParams& p, int i, int& s, int& kvh,
                                            int& part) {
  const int per_part = p.num_seqs * p.num_kv_heads;
  part = i / per_part;
  const int r = i - part * per_part;
  s = r / p.num_kv_heads;
  kvh = r - s * p.num_kv_heads;
}

// A persistent decode worker (THREADS = 160 threads, `tid` 0..159): takes work
// items i = atomicAdd(queue, 1) until i >= num_items (worker_item gives the
// partition, KV head and sequence of i).  Items past a sequence's last
// partition are skipped by the producer.  The ring runs on across items: the
// producer fills each item's first NS positions, and after that every
// consumer warp refills the stage it has just read with its own next
// position of the item (position i + NS of an item is read by the warp that
// read position i), so no warp waits behind a slower one's stage.  Every
// position read is released on its stage's empty barrier, in position order
// per stage; before the producer fills position q it waits until position
// q - NS has been filled (last_fill, written after the release of q - 2NS)
// and then for that position's release, so its parity wait cannot alias a
// phase two back.  Every wait is bounded; a wait that gives up ends the
// worker: the producer stops taking items and loading, the consumers stop at
// the next item, and the producer drains its loads in flight before the
// worker's threads leave (the error word says so).
template <class Tiles, int BS, int NT>
__device__ __forceinline__ void decode_worker(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const DecodeParams& p, uint8_t* smem, int* queue,
                                              int num_items, int tid, uint32_t bar_all,
                                              uint32_t bar_consumers) {
  using Shape = DecodeShape<Tiles, BS, NT>;
  using W = WorkerShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  constexpr int D = Shape::D, NW = Shape::NW, NS = Shape::NS, QD = W::QD, SB = Shape::SB;
  static_assert(NS % NW == 0 && NS * SB <= 32, "refills stay on one warp; one table load per lane");
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + W::BAR_OFF);
  uint64_t* empty_bar = full_bar + NS;
  uint64_t* item_full = empty_bar + NS;
  uint64_t* item_empty = item_full + QD;
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + W::ITEM_OFF);
  volatile int* cur_item = item_slot + QD;
  volatile int* abort = cur_item + 1;
  volatile int* last_fill = abort + 1;  // [NS]: last ring position filled per stage
  float* mg = reinterpret_cast<float*>(smem + W::MERGE_OFF);
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < QD; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 1);
    }
    for (int i = 0; i < NS; ++i) last_fill[i] = -1;
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
    const uint64_t policy = l2_policy_evict_first();
    bool alive = true;
    int g = 0;  // ring position of the next tile
    for (int k = 0;; ++k) {
      int item = -1, s = 0, kvh = 0, part = 0, nblk = 0;
      for (;;) {  // next item with work (a bounded scan of the queue)
        int it = 0;
        if (lane == 0) it = atomicAdd(queue, 1);
        it = __shfl_sync(0xffffffffu, it, 0);
        if (it >= num_items) break;
        worker_item(p, it, s, kvh, part);
        const int L = decode_len<BS>(p, s, lane == 0 && part == 0 && kvh == 0);
        const int nblk_seq = (L + BS - 1) / BS;
        if (part < decode_parts(nblk_seq, p.part_blocks)) {
          item = it;
          nblk = min(p.part_blocks, nblk_seq - part * p.part_blocks);
          break;
        }
      }
      const int slot = k % QD;
      if (lane == 0) {
        if (k >= QD && alive) alive = mbar_wait(&item_empty[slot], ((k / QD) - 1) & 1, abort);
        item_slot[slot] = alive ? item : -1;  // after an abort: tell the consumers to stop
        mbar_arrive(&item_full[slot]);  // release: the consumers' wait acquires item_slot
      }
      alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
      if (item < 0 || !alive) break;
      // the item's first NS positions (its consumers refill the rest)
      const int nstages = (nblk + SB - 1) / SB;
      const int nhead = min(nstages, NS);
      const int32_t* bt = p.block_tables + (size_t)s * p.max_blocks_per_seq + part * p.part_blocks;
      int phys = 0;
      if (lane < nhead * SB && lane < nblk) {
        phys = __ldg(bt + lane);
        if (phys < 0 || phys >= p.num_blocks) {
          record_error(PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
      }
      for (int i = 0; i < nhead; ++i) {
        int ph[SB];
#pragma unroll
        for (int u = 0; u < SB; ++u) ph[u] = __shfl_sync(0xffffffffu, phys, (i * SB + u) & 31);
        if (lane == 0 && alive) {
          const int q = g + i, st = q % NS;
          if (q >= NS) {
            // position q - NS filled (so q - 2NS released), then q - NS released
            const uint64_t t0 = global_timer_ns();
            while (last_fill[st] < q - NS && alive) {
              if (*abort) alive = false;
              else if (global_timer_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                record_error(PA_DEVERR_WAIT_TIMEOUT);
                alive = false;
              }
            }
            if (alive) alive = mbar_wait(&empty_bar[st], ((q / NS) - 1) & 1, abort);
          }
          if (alive) {
            const int nb = min(SB, nblk - i * SB);
            mbar_arrive_expect_tx(&full_bar[st], nb * Shape::BLOCK_BYTES);
            uint8_t* sk = smem + st * Shape::STAGE_BYTES;
#pragma unroll
            for (int u = 0; u < SB; ++u)
              if (u < nb)
                Tiles::issue(sk, sk + Shape::TILE_BYTES, tm_k, tm_v,
                             (ph[u] * p.num_kv_heads + kvh) * BS, u, &full_bar[st], policy);
            last_fill[st] = q;
          }
        }
      }
      alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
      g += nstages;
    }
    named_barrier(bar_all, Shape::THREADS);  // the consumers are done
    if (*abort && lane == 0) {
      // let every load still in flight land before the worker's threads leave
      for (int st = 0; st < NS; ++st)
        if (last_fill[st] >= 0) mbar_drain(&full_bar[st], (last_fill[st] / NS) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const uint64_t policy = l2_policy_evict_first();
  // One thread takes each item from its slot and hands it to all four warps
  // through cur_item, so the warps always agree on the item (and so reach
  // the same named barriers) even if a wait times out.
  int g = 0;
  for (int k = 0;; ++k) {
    if (tid == 0) {
      const int slot = k % QD;
      const bool ok = mbar_wait(&item_full[slot], (k / QD) & 1, abort);
      *cur_item = ok ? item_slot[slot] : -1;
      mbar_arrive(&item_empty[slot]);
    }
    __syncwarp();
    named_barrier(bar_consumers, NW * 32);
    const int item = *cur_item;
    if (item < 0) break;
    int s, kvh, part;
    worker_item(p, item, s, kvh, part);
    const int L = decode_len<BS>(p, s, false);
    const int nblk_seq = (L + BS - 1) / BS;
    const int nparts = decode_parts(nblk_seq, p.part_blocks);
    const int blk0 = part * p.part_blocks;
    const int nblk = min(p.part_blocks, nblk_seq - blk0);
    uint32_t qf[D / 16][NT][2];
    static_assert(Shape::HP == 1, "the mixed batch's decode workers read one KV head per item");
    Tiles::template load_q<NT>(
        qf, reinterpret_cast<const T*>(p.query) +
                ((size_t)s * p.num_q_heads + (size_t)kvh * p.group) * D,
        p.group, lane);
    float m_run[NT][2], l_run[NT][2];
    float o[D / 16][NT][4];
    reset_state<Tiles, NT>(o, m_run, l_run);
    const int nstages = (nblk + Shape::SB - 1) / Shape::SB;
    // a stage may reach past the item's last block (into the next partition)
    const int L_end = min(L, (blk0 + nblk) * BS);
    bool alive = true;
    const int32_t* bt = p.block_tables + (size_t)s * p.max_blocks_per_seq + blk0;
    int ids[SB];  // lane l: the blocks of this warp's (kw + l)-th position of the item
    int kw = -32;
    for (int i = warp; i < nstages; i += NW) {
      const int gi = g + i, st = gi % NS;
      // after a wait gave up the warp still runs through its (garbage) stages,
      // every lane alike, so the .aligned loads and MMAs stay converged
      if (alive) alive = mbar_wait(&full_bar[st], (gi / NS) & 1, abort);
      consume_block<Tiles, BS, NT>(o, m_run, l_run, qf, smem + st * Shape::STAGE_BYTES,
                                   (blk0 + i * SB) * BS, L_end, p.scale_log2, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
      const int nxt = i + NS;  // this warp's next position on stage st (warp-uniform test)
      if (nxt < nstages) {
        const int kk = (nxt - warp) / NW;
        if (kk >= kw + 32) {
          kw = kk;
#pragma unroll
          for (int u = 0; u < SB; ++u) {
            const int b = (warp + NW * (kk + lane)) * SB + u;
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
        for (int u = 0; u < SB; ++u) ph[u] = __shfl_sync(0xffffffffu, ids[u], kk - kw);
        if (lane == 0 && alive) {
          // the warp's reads of the stage are done (__syncwarp above); order
          // them before the async-proxy writes that refill it
          fence_proxy_async_smem();
          const int nb = min(SB, nblk - nxt * SB);
          mbar_arrive_expect_tx(&full_bar[st], nb * Shape::BLOCK_BYTES);
          uint8_t* sk = smem + st * Shape::STAGE_BYTES;
#pragma unroll
          for (int u = 0; u < SB; ++u)
            if (u < nb)
              Tiles::issue(sk, sk + Shape::TILE_BYTES, tm_k, tm_v,
                           (ph[u] * p.num_kv_heads + kvh) * BS, u, &full_bar[st], policy);
          // the release of gi above is visible before this position is
          __threadfence_block();
          last_fill[st] = g + nxt;
        }
      }
    }
    g += nstages;
    // the opening barrier of merge_item also orders this item's read of
    // cur_item before thread 0 overwrites it for the next item
    merge_item_two_pass<Tiles, BS, NT>(mg, o, m_run, l_run, p, s, kvh, part, nparts == 1, tid,
                                       bar_consumers);
  }
  named_barrier(bar_all, Shape::THREADS);  // lets the producer see the final abort word
}

// CTA shape of the mixed launch.  With one query n-tile (groups up to 8) a
// CTA of 16 warps hosts three decode workers, 12 consumer warps per SM as
// three pa_decode CTAs have, and a prefill tile's softmax warpgroups get 200
// registers, its producer warpgroup 88 and the idle fourth warpgroup 24
// (2 x 128 x 200 + 128 x 88 + 128 x 24 = 512 x 128).  With two n-tiles the
// consumers need more registers: 12 warps and two workers.
template <typename T, int BS, int NT>
struct MixedShape {
  using Pf = PrefillShape<T, BS>;
  using Tiles = HalfTiles<T, 128, BS>;
  using Dc = DecodeShape<Tiles, BS, NT>;
  using Wk = WorkerShape<Tiles, BS, NT>;
  static constexpr int THREADS = NT == 1 ? 512 : Pf::THREADS;
  static constexpr int WORKERS = THREADS / Dc::THREADS;  // decode workers per CTA
  static constexpr uint32_t SOFT_REGS = Pf::SOFTMAX_REGS;
  static constexpr uint32_t PROD_REGS = NT == 1 ? 88 : Pf::PRODUCER_REGS;
  static constexpr uint32_t IDLE_REGS = NT == 1 ? 24 : PROD_REGS;  // warps 12-15
  static constexpr int MIN_LAUNCH_REGS = NT == 1 ? 128 : Pf::MIN_LAUNCH_REGS;
  static_assert(2 * 128 * SOFT_REGS + 128 * PROD_REGS + (THREADS - 384) * IDLE_REGS <=
                    THREADS * MIN_LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static constexpr int DEC_SMEM = 1024 + WORKERS * Wk::BYTES;
  static constexpr int SMEM_BYTES = Pf::SMEM_BYTES > DEC_SMEM ? Pf::SMEM_BYTES : DEC_SMEM;
  static_assert(WORKERS == (NT == 1 ? 3 : 2), "decode workers per CTA");
  static_assert(1 + 2 * WORKERS <= 16, "named barrier ids");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
};

// Launch order of the mixed grid (every count even: CTA pairs share a TPC):
//   [0, lead)                          prefill slots 0 .. lead - 1
//   [lead, lead + early)               decode CTAs started with the first tiles
//   [lead + early, prefill_slots + early)  prefill slots lead ..
//   [prefill_slots + early, grid)      decode CTAs that start as the tiles end
struct MixedPlan {
  int prefill_ctas;       // prefill tiles
  int prefill_slots;      // prefill_ctas rounded up to even
  int lead;               // prefill slots launched before the early decode CTAs
  int early;              // decode CTAs launched with the first prefill tiles
  int prefill_tiles;      // 256-row tiles per prefill sequence (from max_q_len)
  int first_prefill_seq;  // == number of decode sequences
  int decode_items;       // num_decode * num_kv_heads * max_parts
  int* queue;             // decode work-item counter, zero at launch
};

template <typename T, int BS, int NT>
__global__ void __launch_bounds__(MixedShape<T, BS, NT>::THREADS, 1)
    mixed_kernel(const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, PrefillParams pp, DecodeParams dp,
                 MixedPlan plan) {
  using Sh = MixedShape<T, BS, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // the split-KV combine that follows may be launched (it waits for this grid)
  griddep_launch_dependents();
  const int b = blockIdx.x;
  const bool is_early = b >= plan.lead && b < plan.lead + plan.early;
  // prefill slot of this CTA, or its index among the decode CTAs
  const int slot = b < plan.lead ? b : b - plan.early;
  if (!is_early && slot < plan.prefill_slots) {
    if (slot >= plan.prefill_ctas) return;  // the spare slot of an odd count
    // per chunk, the tile that sees the most keys first; query heads h and
    // h + 1 of one tile side by side, so a CTA pair (one TPC) runs two
    // tiles of the same length over the same K/V
    const int h = slot % pp.num_q_heads;
    const int rest = slot / pp.num_q_heads;
    const int tile = plan.prefill_tiles - 1 - rest % plan.prefill_tiles;
    const int s = plan.first_prefill_seq + rest / plan.prefill_tiles;
    prefill_tile<T, BS, Sh::SOFT_REGS, Sh::PROD_REGS, 128, Sh::IDLE_REGS>(&tm_q, &tm_k, &tm_v, pp,
                                                                          smem, tile, h, s);
    return;
  }
  const int w = threadIdx.x / Sh::Dc::THREADS;
  if (w >= Sh::WORKERS) return;  // the spare warps
  const int tid = threadIdx.x - w * Sh::Dc::THREADS;
  // decode rows: sequence s must own exactly query row s
  if (w == 0 && tid == 0) {
    const int nd = plan.first_prefill_seq;
    const int d = is_early ? b - plan.lead : b - plan.prefill_slots;  // decode CTA index
    for (int s = d; s < nd; s += gridDim.x - plan.prefill_slots)
      if (pp.cu_q_lens[s] != s || pp.cu_q_lens[s + 1] != s + 1) record_error(PA_DEVERR_SEQ_RANGE);
  }
  decode_worker<typename Sh::Tiles, BS, NT>(&tm_k, &tm_v, dp, smem + w * Sh::Wk::BYTES,
                                            plan.queue, plan.decode_items, tid, 1 + w,
                                            1 + Sh::WORKERS + w);
}

}  // namespace pa
