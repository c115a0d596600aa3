// pa_api.cu — the extern "C" boundary of libpa.so (declared in include/pa.h):
// argument validation, split-KV partition planning, TMA tensor-map encoding
// and template dispatch onto the sm_100a kernels.  Nothing here allocates
// device memory or synchronises (except pa_get_device_error).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <type_traits>
#include <climits>
#include <cmath>
#include <mutex>

#include "../../include/pa.h"
#include "cache_ops.cuh"
#include "decode.cuh"
#include "mixed.cuh"
#include "prefill.cuh"

namespace {

constexpr int kVersion = (1 << 16) | 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library links no libcuda at build time and loads on machines without a GPU.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major [rows][cols] tensor with a row pitch of `pitch_elems`, boxes of
// {128 bytes of columns, box_rows rows}, 128-byte swizzle.
bool make_map_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t pitch_elems, uint32_t box_rows, pa_dtype dt) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t esize = dt == PA_FP8_E4M3 ? 1 : 2;
  const CUtensorMapDataType type = dt == PA_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_elems * esize};
  cuuint32_t box[2] = {128 / esize, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool valid_dtype(pa_dtype d) { return d == PA_F16 || d == PA_BF16; }
bool valid_cache_dtype(pa_dtype d) { return valid_dtype(d) || d == PA_FP8_E4M3; }

// Split-KV scratch for pa_decode_static_workspace, for callers that cannot
// allocate: one array per device, part of the module's own device memory.
// Host code must not pass the symbol itself to a kernel (on the host it is a
// stand-in, not a device address); static_workspace_address resolves the real
// address once per device, with that device current, and caches it.
static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
int sm_count() {
  static std::atomic<int> cached[kMaxDevices];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);  // every thread stores the same value
  }
  return n;
}

// One-time per (kernel, device) launch configuration: the dynamic shared
// memory limit is a per-device function attribute, so a process that drives
// several GPUs must set it on each.  `done` is the caller's per-kernel flag
// word (bit d: device d configured): kernel instantiations share a function
// type, so the flags cannot live in this template.  `min_regs` > 0 also
// refuses a build whose kernel has fewer registers per thread than its
// setmaxnreg split needs (the register increase could never be granted).
template <typename K>
pa_status configure_kernel(std::atomic<unsigned long long>& done, K kern, int smem_bytes,
                           int min_regs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  const unsigned long long bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return PA_OK;
  if (min_regs > 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return PA_ERR_CUDA;
    if (attr.numRegs < min_regs) return PA_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_release);
  return PA_OK;
}

std::mutex g_static_ws_mutex;
void* g_static_ws_addr[kMaxDevices] = {};

pa_status static_workspace_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (g_static_ws_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    g_static_ws_addr[dev] = p;
  }
  *addr = g_static_ws_addr[dev];
  return PA_OK;
}

// Split-KV partition length in tokens.  Partitions are whole blocks; the aim
// is several waves of CTAs over the device's SMs while keeping each partition
// long enough (>= 256 tokens) that its fixed cost and its partial write stay
// small.  The choice depends only on sizes and the SM count, never on data.
int auto_partition_tokens(int num_seqs, int num_kv_heads, int block_size, int max_seq_len) {
  const long long units = (long long)num_seqs * num_kv_heads;
  const long long target_ctas = (long long)sm_count() * 3 * 8;  // ~8 waves at 3 CTAs per SM
  long long per = (long long)max_seq_len * units / target_ctas;
  int p = 256;
  while (p < 2048 && p < per) p *= 2;
  if (p < block_size) p = block_size;
  return (p / block_size) * block_size;
}

// A caller's partition length rounded up to whole blocks; lengths above 2^30
// tokens are clamped there first (any partition longer than every sequence
// means one partition), so the rounding cannot overflow.
int round_partition_tokens(int requested, int block_size) {
  const long long r = requested > (1 << 30) ? (1 << 30) : requested;
  return (int)(((r + block_size - 1) / block_size) * block_size);
}

int partition_tokens_for(int requested, int num_seqs, int num_kv_heads, int block_size,
                         int max_seq_len) {
  if (requested > 0) return round_partition_tokens(requested, block_size);
  return auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_seq_len);
}

// Partitions of a sequence of `len` tokens (at least one).
long long num_partitions(int len, int pt) { return len == 0 ? 1 : ((long long)len + pt - 1) / pt; }

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream still runs (from the moment all of that
// kernel's CTAs have executed griddepcontrol.launch_dependents); it must
// itself wait (griddepcontrol.wait) before it reads what that kernel writes.
template <typename... KArgs, typename... Args>
pa_status launch_overlapped(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? PA_OK
                                                                                    : PA_ERR_CUDA;
}

// The split-KV combine after a decode launch, launched to overlap its tail
// (decode_reduce_kernel waits for the decode grid before reading partials).
template <typename T, int D>
pa_status launch_combine(const pa::DecodeParams& p, int block_size, cudaStream_t stream) {
  const int units = p.num_seqs * p.num_q_heads;
  return launch_overlapped(pa::decode_reduce_kernel<T, D>,
                           dim3((units + pa::REDUCE_WARPS - 1) / pa::REDUCE_WARPS),
                           dim3(pa::REDUCE_WARPS * 32), 0, stream, p, block_size);
}

template <class Tiles, int BS, int NT>
pa_status run_decode(const CUtensorMap& mk, const CUtensorMap& mv, pa::DecodeParams p,
                     int num_parts, cudaStream_t stream) {
  using Shape = pa::DecodeShape<Tiles, BS, NT>;
  using T = typename Tiles::Elem;
  auto kern = pa::decode_kernel<Tiles, BS, NT>;
  static std::atomic<unsigned long long> configured{0};  // per instantiation
  if (pa_status st = configure_kernel(configured, kern, Shape::SMEM_BYTES, 0); st != PA_OK)
    return st;
  dim3 grid(num_parts, p.num_kv_heads / Tiles::HP, p.num_seqs);  // y: packs of HP kv heads
  kern<<<grid, Shape::THREADS, Shape::SMEM_BYTES, stream>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (num_parts > 1) return launch_combine<T, Shape::D>(p, BS, stream);
  return PA_OK;
}

// Shared-prefix decode: the prefix partitions [0, n_prefix) of every
// sequence in prefix_decode_kernel (one CTA per partition, KV head and group
// of p.seq_group sequences), the remaining partitions [n_prefix, num_parts)
// in decode_kernel, then the combine.
template <typename T, int BS>
pa_status run_shared_prefix(const CUtensorMap& mk, const CUtensorMap& mv, pa::DecodeParams p,
                            int num_parts, int n_prefix, cudaStream_t stream) {
  using Tiles = pa::HalfTiles<T, 128, BS>;
  using Shape = pa::DecodeShape<Tiles, BS, 2>;
  auto kern = pa::prefix_decode_kernel<Tiles, BS>;
  static std::atomic<unsigned long long> configured{0};
  if (pa_status st = configure_kernel(configured, kern, Shape::SMEM_BYTES, 0); st != PA_OK)
    return st;
  const int groups = (p.num_seqs + p.seq_group - 1) / p.seq_group;
  kern<<<dim3(n_prefix, p.num_kv_heads, groups), Shape::THREADS, Shape::SMEM_BYTES, stream>>>(
      mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (num_parts > n_prefix) {
    // the other partitions overlap the prefix pass: they write other
    // partials and wait for the prefix grid before their own grid ends
    p.part_base = n_prefix;
    auto launch = [&](auto nt_tag) -> pa_status {
      constexpr int NT = decltype(nt_tag)::value;
      using S = pa::DecodeShape<Tiles, BS, NT>;
      auto dk = pa::decode_kernel<Tiles, BS, NT>;
      static std::atomic<unsigned long long> conf{0};
      if (pa_status st = configure_kernel(conf, dk, S::SMEM_BYTES, 0); st != PA_OK) return st;
      return launch_overlapped(dk, dim3(num_parts - n_prefix, p.num_kv_heads, p.num_seqs),
                               dim3(S::THREADS), S::SMEM_BYTES, stream, mk, mv, p);
    };
    const pa_status st = p.group <= 8 ? launch(std::integral_constant<int, 1>{})
                                      : launch(std::integral_constant<int, 2>{});
    if (st != PA_OK) return st;
  }
  if (num_parts > 1) return launch_combine<T, 128>(p, BS, stream);
  return PA_OK;
}

template <class Tiles, int BS>
pa_status dispatch_group(const CUtensorMap& mk, const CUtensorMap& mv, pa::DecodeParams p,
                         int num_parts, cudaStream_t stream) {
  if (p.group <= 8) return run_decode<Tiles, BS, 1>(mk, mv, p, num_parts, stream);
  return run_decode<Tiles, BS, 2>(mk, mv, p, num_parts, stream);
}

template <typename T>
pa_status dispatch_decode(int D, int BS, const CUtensorMap& mk, const CUtensorMap& mv,
                          pa::DecodeParams p, int num_parts, cudaStream_t stream) {
  using namespace pa;
  if (D == 128 && BS == 16) return dispatch_group<HalfTiles<T, 128, 16>, 16>(mk, mv, p, num_parts, stream);
  if (D == 128 && BS == 32) return dispatch_group<HalfTiles<T, 128, 32>, 32>(mk, mv, p, num_parts, stream);
  if (D == 64 && BS == 16) return dispatch_group<HalfTiles<T, 64, 16>, 16>(mk, mv, p, num_parts, stream);
  if (D == 64 && BS == 32) return dispatch_group<HalfTiles<T, 64, 32>, 32>(mk, mv, p, num_parts, stream);
  return PA_ERR_UNSUPPORTED;
}

// FP8 head packing: with 16-token blocks, two adjacent kv heads share a ring
// stage (one contiguous 4 KB box) whenever their query heads fit one 8-wide
// n-tile; the tensor maps' boxes must then be 2 x 16 rows high.
bool fp8_pack_heads(int block_size, int group, int num_kv_heads) {
  return block_size == 16 && 2 * group <= 8 && num_kv_heads % 2 == 0;
}

template <typename T>
pa_status dispatch_decode_fp8(int BS, const CUtensorMap& mk, const CUtensorMap& mv,
                              pa::DecodeParams p, int num_parts, cudaStream_t stream) {
  using namespace pa;
  if (BS == 16 && fp8_pack_heads(BS, p.group, p.num_kv_heads))
    return run_decode<E4m3Tiles<T, 16, 2>, 16, 1>(mk, mv, p, num_parts, stream);
  if (BS == 16) return dispatch_group<E4m3Tiles<T, 16>, 16>(mk, mv, p, num_parts, stream);
  if (BS == 32) return dispatch_group<E4m3Tiles<T, 32>, 32>(mk, mv, p, num_parts, stream);
  return PA_ERR_UNSUPPORTED;
}

// Workspace of pa_prefill_chunk: 256 bytes of alignment slack, 1 KB of
// per-unit counters, then the partial rows of up to two waves (2 x #SMs) of
// split parts: O [parts][256][D] and (m, l) [parts][256][2], fp32.
constexpr size_t kPrefillCounterBytes = 1024;
constexpr int kPrefillPartWaves = 2;
size_t prefill_workspace_bytes(int head_dim) {
  return 256 + kPrefillCounterBytes +
         (size_t)kPrefillPartWaves * sm_count() * 256 * (head_dim + 2) * sizeof(float);
}

// Tail split plan.  Work units (256 rows of a query head of a sequence) run
// one CTA per SM (the kernel uses all of tensor memory), so `units` take
// ceil(units / #SMs) waves of about one unit's time each.  The last
// rem = units mod #SMs units can be cut into k parts along the key range;
// their rem * k parts then take ceil(rem * k / #SMs) waves of 1/k of a unit.
// The plan takes the k in 2..4 that minimises that (the smallest on ties),
// if it beats one whole wave and the parts fit the workspace.
void plan_prefill_split(pa::PrefillParams& p, long long units, bool have_ws) {
  const int nsm = sm_count();
  const long long rem = units % nsm;
  int best_k = 1;
  double best_t = 1.0;
  for (int k = 2; k <= 4 && have_ws && rem > 0; ++k) {
    if (rem * k > (long long)kPrefillPartWaves * nsm) break;
    const double t = (double)((rem * k + nsm - 1) / nsm) / k;
    if (t < best_t - 1e-9) {
      best_t = t;
      best_k = k;
    }
  }
  if (rem > (long long)(kPrefillCounterBytes / sizeof(int))) best_k = 1;
  p.split = best_k;
  p.n_full = (int)(best_k > 1 ? units - rem : units);
}

template <typename T, int BS, int D>
pa_status run_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      pa::PrefillParams p, cudaStream_t stream) {
  using Sh = pa::PrefillShape<T, BS, D>;
  auto kern = pa::prefill_kernel<T, BS, D>;
  // the kernel's setmaxnreg split assumes at least MIN_LAUNCH_REGS registers per thread
  static std::atomic<unsigned long long> configured{0};  // per instantiation
  if (pa_status st = configure_kernel(configured, kern, Sh::SMEM_BYTES, Sh::MIN_LAUNCH_REGS);
      st != PA_OK)
    return st;
  const long long units = (long long)p.tiles_per_seq * p.num_q_heads * p.num_seqs;
  const long long grid = p.n_full + (units - p.n_full) * p.split;
  if (grid > INT_MAX) return PA_ERR_INVALID_ARG;
  if (p.split > 1 &&
      cudaMemsetAsync(p.counters, 0, (units - p.n_full) * sizeof(int), stream) != cudaSuccess)
    return PA_ERR_CUDA;
  kern<<<(unsigned)grid, Sh::THREADS, Sh::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  return launch_status();
}

template <typename T, int D>
pa_status dispatch_prefill_bs(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const pa::PrefillParams& p, int block_size, cudaStream_t st) {
  if (block_size == 16) return run_prefill<T, 16, D>(mq, mk, mv, p, st);
  return run_prefill<T, 32, D>(mq, mk, mv, p, st);
}
pa_status dispatch_prefill(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const pa::PrefillParams& p, pa_dtype dtype, int block_size,
                           int head_dim, cudaStream_t st) {
  if (dtype == PA_BF16)
    return head_dim == 64 ? dispatch_prefill_bs<__nv_bfloat16, 64>(mq, mk, mv, p, block_size, st)
                          : dispatch_prefill_bs<__nv_bfloat16, 128>(mq, mk, mv, p, block_size, st);
  return head_dim == 64 ? dispatch_prefill_bs<__half, 64>(mq, mk, mv, p, block_size, st)
                        : dispatch_prefill_bs<__half, 128>(mq, mk, mv, p, block_size, st);
}

// Split-KV partition length of the decode rows of a mixed batch: as for
// pa_decode, capped at 1024 tokens so that the decode workers' queue ends in
// short items (the last item of a worker bounds how long it idles at the end).
int mixed_partition_tokens(int requested, int num_decode, int num_kv_heads, int block_size,
                           int max_dec_len) {
  if (requested > 0) return round_partition_tokens(requested, block_size);
  const int p = auto_partition_tokens(num_decode, num_kv_heads, block_size, max_dec_len);
  return p > 1024 ? 1024 : p;
}

// Bytes of a mixed batch's workspace: 256 of alignment slack, the 256-byte
// queue-counter block, then the decode rows' split-KV partials.
size_t mixed_workspace_bytes(int num_decode, int num_q_heads, int head_dim, int num_parts) {
  if (num_decode <= 0) return 0;
  size_t b = 512;
  if (num_parts > 1) b += (size_t)num_decode * num_q_heads * num_parts * (head_dim + 2) * sizeof(float);
  return b;
}


// Share of the SMs the first prefill tiles of a mixed launch take (the rest
// start decode workers).  Tuned on B200 for 256 decode rows over U[128, 4096]
// cached tokens beside four 512-row chunks over 8192 cached tokens: prefill
// there is ~58 % of the launch's SM time when decode runs at the SMs'
// unsaturated rate.
constexpr double kMixedPrefillShare = 7.0 / 12.0;

template <typename T, int BS, int NT>
pa_status run_mixed(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const pa::PrefillParams& pp, const pa::DecodeParams& dp,
                    const pa::MixedPlan& plan, cudaStream_t stream) {
  using Sh = pa::MixedShape<T, BS, NT>;
  auto kern = pa::mixed_kernel<T, BS, NT>;
  // same register-split requirement as prefill_kernel (its prefill tiles
  // run the same setmaxnreg split)
  static std::atomic<unsigned long long> configured{0};  // per instantiation
  if (pa_status st = configure_kernel(configured, kern, Sh::SMEM_BYTES, Sh::MIN_LAUNCH_REGS);
      st != PA_OK)
    return st;
  // persistent decode workers: at most one CTA per SM; clusters of two CTAs
  // (one TPC each), so every count is even
  const int n_sm = sm_count() & ~1;
  long long decode_ctas = ((long long)plan.decode_items + Sh::WORKERS - 1) / Sh::WORKERS;
  if (decode_ctas > n_sm) decode_ctas = n_sm;
  decode_ctas = (decode_ctas + 1) & ~1LL;
  const long long grid = plan.prefill_slots + decode_ctas;
  // The first prefill tiles take kMixedPrefillShare of the SMs and decode
  // workers start on the rest at once, so the HBM-bound decode runs beside the
  // tensor-bound tiles; later tiles follow on the SMs the first ones free, and
  // the remaining decode CTAs start as the tiles run out (decode workers that
  // find the queue empty exit, handing their SMs to the next tiles).
  pa::MixedPlan pl = plan;
  pl.lead = (int)std::min<long long>(plan.prefill_slots,
                                     (long long)(n_sm * kMixedPrefillShare) & ~1LL);
  pl.early = (int)std::min<long long>(decode_ctas, n_sm - pl.lead);
  if (grid <= 0) return PA_OK;
  if (grid > INT_MAX) return PA_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(Sh::THREADS);
  cfg.dynamicSmemBytes = Sh::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, pp, dp, pl) != cudaSuccess) return PA_ERR_CUDA;
  if (plan.decode_items > 0 && dp.max_parts > 1) return launch_combine<T, 128>(dp, BS, stream);
  return PA_OK;
}

template <typename T, int BS>
pa_status dispatch_mixed(int group, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const pa::PrefillParams& pp,
                         const pa::DecodeParams& dp, const pa::MixedPlan& plan,
                         cudaStream_t stream) {
  if (group <= 8) return run_mixed<T, BS, 1>(mq, mk, mv, pp, dp, plan, stream);
  return run_mixed<T, BS, 2>(mq, mk, mv, pp, dp, plan, stream);
}

// Self-test of the bounded waits (pa_selftest_wait_timeout): two roles of one
// CTA wait on mbarriers that nothing ever arrives on.  Role 0 (warp 0) gives
// up after `limit_ns`; role 1 (warp 1) has the kernels' normal limit but polls
// the CTA's abort word, which role 0 sets, so it gives up right after.  Each
// role writes how long it waited.  No memory but the two words is touched.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, uint64_t* waited_ns) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_word;
  volatile int* abort = &abort_word;
  if (threadIdx.x == 0) {
    pa::mbar_init(&bars[0], 1);
    pa::mbar_init(&bars[1], 1);
    *abort = 0;
    pa::fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t t0 = pa::global_timer_ns();
    pa::mbar_wait(&bars[warp], 0, abort, warp == 0 ? limit_ns : pa::kWaitLimitNs);
    if (waited_ns != nullptr) waited_ns[warp] = pa::global_timer_ns() - t0;
  }
}

}  // namespace

extern "C" {

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_OUT_OF_RANGE: return "PA_ERR_OUT_OF_RANGE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    default: return "PA_ERR_UNKNOWN";
  }
}

int pa_version(void) { return kVersion; }

pa_status pa_slot_mapping(int64_t* slot_mapping, const int32_t* block_tables,
                          const int32_t* cu_q_lens, const int32_t* ctx_lens, int num_seqs,
                          int num_tokens, int max_blocks_per_seq, int block_size,
                          pa_stream_t stream) {
  if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (num_seqs == 0 || !slot_mapping || !block_tables || !ctx_lens) return PA_ERR_INVALID_ARG;
  if (cu_q_lens == nullptr && num_tokens != num_seqs) return PA_ERR_INVALID_ARG;
  const int threads = 256;
  pa::slot_mapping_kernel<<<(num_tokens + threads - 1) / threads, threads, 0,
                            (cudaStream_t)stream>>>(slot_mapping, block_tables, cu_q_lens,
                                                    ctx_lens, num_seqs, num_tokens,
                                                    max_blocks_per_seq, block_size);
  return launch_status();
}

pa_status pa_reshape_and_cache(const void* key, const void* value, void* key_cache,
                               void* value_cache, const int64_t* slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               pa_dtype dtype, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  const long long total = (long long)num_tokens * num_kv_heads * (head_dim * 2 / 16);
  const int threads = 256;
  const long long grid = (total + threads - 1) / threads;
  if (grid > INT_MAX) return PA_ERR_INVALID_ARG;
  const int64_t num_slots = (int64_t)num_blocks * block_size;
  auto st = (cudaStream_t)stream;
  auto k = reinterpret_cast<const uint4*>(key);
  auto v = reinterpret_cast<const uint4*>(value);
  auto kc = reinterpret_cast<uint4*>(key_cache);
  auto vc = reinterpret_cast<uint4*>(value_cache);
  if (head_dim == 128)
    pa::reshape_and_cache_kernel<128><<<(unsigned)grid, threads, 0, st>>>(
        k, v, kc, vc, slot_mapping, num_tokens, num_kv_heads, block_size, num_slots);
  else if (head_dim == 64)
    pa::reshape_and_cache_kernel<64><<<(unsigned)grid, threads, 0, st>>>(
        k, v, kc, vc, slot_mapping, num_tokens, num_kv_heads, block_size, num_slots);
  else
    return PA_ERR_UNSUPPORTED;
  return launch_status();
}

pa_status pa_append(const void* key, const void* value, void* key_cache, void* value_cache,
                    const int32_t* block_tables, const int32_t* cu_q_lens, const int32_t* ctx_lens,
                    int64_t* slot_mapping, int num_seqs, int num_tokens, int max_blocks_per_seq,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                    pa_stream_t stream) {
  if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || !valid_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (num_seqs == 0 || !key || !value || !key_cache || !value_cache || !block_tables ||
      !ctx_lens)
    return PA_ERR_INVALID_ARG;
  if (cu_q_lens == nullptr && num_tokens != num_seqs) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  const long long total = (long long)num_tokens * num_kv_heads * (head_dim * 2 / 16);
  const int threads = 256;
  const long long grid = (total + threads - 1) / threads;
  if (grid > INT_MAX) return PA_ERR_INVALID_ARG;
  auto st = (cudaStream_t)stream;
  auto k = reinterpret_cast<const uint4*>(key);
  auto v = reinterpret_cast<const uint4*>(value);
  auto kc = reinterpret_cast<uint4*>(key_cache);
  auto vc = reinterpret_cast<uint4*>(value_cache);
  if (head_dim == 128)
    pa::append_kernel<128><<<(unsigned)grid, threads, 0, st>>>(
        k, v, kc, vc, block_tables, cu_q_lens, ctx_lens, slot_mapping, num_seqs, num_tokens,
        num_kv_heads, max_blocks_per_seq, block_size, num_blocks);
  else if (head_dim == 64)
    pa::append_kernel<64><<<(unsigned)grid, threads, 0, st>>>(
        k, v, kc, vc, block_tables, cu_q_lens, ctx_lens, slot_mapping, num_seqs, num_tokens,
        num_kv_heads, max_blocks_per_seq, block_size, num_blocks);
  else
    return PA_ERR_UNSUPPORTED;
  return launch_status();
}

pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_cache_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_pairs) return PA_ERR_INVALID_ARG;
  if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_INVALID_ARG;
  const int64_t block_bytes =
      (int64_t)num_kv_heads * block_size * head_dim * (dtype == PA_FP8_E4M3 ? 1 : 2);
  if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
  const int64_t chunks = block_bytes / 16;
  pa::copy_blocks_kernel<8><<<dim3(num_pairs, 2), 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<uint4*>(key_cache), reinterpret_cast<uint4*>(value_cache), block_pairs,
      chunks, num_blocks);
  return launch_status();
}

pa_status pa_swap_blocks(void* dst_key_cache, void* dst_value_cache, const void* src_key_cache,
                         const void* src_value_cache, const int64_t* block_pairs, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int src_num_blocks,
                         int dst_num_blocks, pa_dtype dtype, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      src_num_blocks <= 0 || dst_num_blocks <= 0 || !valid_cache_dtype(dtype))
    return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || !block_pairs)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(dst_key_cache) || !aligned16(dst_value_cache) || !aligned16(src_key_cache) ||
      !aligned16(src_value_cache))
    return PA_ERR_INVALID_ARG;
  const int64_t block_bytes =
      (int64_t)num_kv_heads * block_size * head_dim * (dtype == PA_FP8_E4M3 ? 1 : 2);
  if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
  pa::swap_blocks_kernel<8><<<dim3(num_pairs, 2), 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<uint4*>(dst_key_cache), reinterpret_cast<uint4*>(dst_value_cache),
      reinterpret_cast<const uint4*>(src_key_cache), reinterpret_cast<const uint4*>(src_value_cache),
      block_pairs, block_bytes / 16, src_num_blocks, dst_num_blocks);
  return launch_status();
}

int pa_decode_partition_tokens(int num_seqs, int num_kv_heads, int block_size, int max_seq_len) {
  if (num_seqs <= 0 || num_kv_heads <= 0 || block_size <= 0 || max_seq_len < 0) return 0;
  return auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_seq_len);
}

pa_status pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int block_size, int max_seq_len, int partition_tokens,
                                   size_t* bytes) {
  if (!bytes || num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_seq_len < 0 || partition_tokens < 0)
    return PA_ERR_INVALID_ARG;
  const int pt = partition_tokens_for(partition_tokens, num_seqs, num_kv_heads, block_size,
                                      max_seq_len);
  const long long parts = num_partitions(max_seq_len, pt);
  if (parts <= 1) {
    *bytes = 0;
    return PA_OK;
  }
  *bytes = (size_t)num_seqs * num_q_heads * parts * (head_dim + 2) * sizeof(float) + 256;
  return PA_OK;
}

}  // extern "C"

namespace {

// Validation, partition planning and launch shared by pa_decode (fp16 / bf16
// caches) and pa_decode_fp8 (E4M3 caches, kv_fp8 = true).
// The fused append of pa_append_decode (null for plain decode).
struct AppendArgs {
  const void* new_key;
  const void* new_value;
  int64_t* slot_out;
};

// The shared prefix of pa_decode_shared_prefix (null for the other calls).
struct PrefixArgs {
  const int32_t* blocks;
  int len;  // tokens, a multiple of block_size
};

pa_status decode_impl(void* out, const void* query, const void* key_cache,
                      const void* value_cache, const int32_t* block_tables,
                      const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                      int max_seq_len, int partition_tokens, float scale, float k_scale,
                      float v_scale, bool kv_fp8, pa_dtype dtype, void* workspace,
                      size_t workspace_bytes, pa_stream_t stream,
                      const AppendArgs* app = nullptr, const PrefixArgs* prefix = nullptr) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || max_seq_len < 0 || partition_tokens < 0 ||
      !valid_dtype(dtype) || !std::isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (kv_fp8 && !(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) &&
                  v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if (app && (!app->new_key || !app->new_value || !aligned16(app->new_key) ||
              !aligned16(app->new_value)))
    return PA_ERR_INVALID_ARG;
  if ((long long)max_seq_len > (long long)max_blocks_per_seq * block_size)
    return PA_ERR_INVALID_ARG;
  if (prefix && (prefix->len < 0 || (prefix->len > 0 && prefix->blocks == nullptr) ||
                 block_size <= 0 || prefix->len % block_size != 0 || prefix->len > max_seq_len))
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 65535) return PA_ERR_INVALID_ARG;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (kv_fp8 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if ((long long)num_blocks * num_kv_heads * block_size > INT_MAX) return PA_ERR_INVALID_ARG;

  const int pt = partition_tokens_for(partition_tokens, num_seqs, num_kv_heads, block_size,
                                      max_seq_len);
  const long long parts = num_partitions(max_seq_len, pt);
  if (parts > 65535) return PA_ERR_INVALID_ARG;
  const int num_parts = (int)parts;
  size_t need = 0;
  pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_seq_len, partition_tokens, &need);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return PA_ERR_WORKSPACE;

  CUtensorMap mk, mv;
  const uint64_t rows = (uint64_t)num_blocks * num_kv_heads * block_size;
  const pa_dtype cache_dt = kv_fp8 ? PA_FP8_E4M3 : dtype;
  const uint32_t box_rows =
      kv_fp8 && fp8_pack_heads(block_size, num_q_heads / num_kv_heads, num_kv_heads)
          ? 2 * block_size
          : block_size;
  if (!make_map_2d(&mk, key_cache, head_dim, rows, head_dim, box_rows, cache_dt) ||
      !make_map_2d(&mv, value_cache, head_dim, rows, head_dim, box_rows, cache_dt))
    return PA_ERR_CUDA;

  pa::DecodeParams p;
  p.out = out;
  p.query = query;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  float* ws = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  const size_t acc_elems = (size_t)num_seqs * num_q_heads * num_parts * head_dim;
  p.ws_acc = need > 0 ? ws : nullptr;
  p.ws_ml = need > 0 ? ws + acc_elems : nullptr;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.num_blocks = num_blocks;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.part_blocks = pt / block_size;
  p.max_parts = num_parts;
  p.scale_log2 = scale * (kv_fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  p.v_scale = kv_fp8 ? v_scale : 1.f;
  p.k_scale = kv_fp8 ? k_scale : 1.f;
  p.len_add = app ? 1 : 0;  // fused append: seq_lens holds the context lengths
  p.new_key = app ? app->new_key : nullptr;
  p.new_value = app ? app->new_value : nullptr;
  p.key_cache = app ? const_cast<void*>(key_cache) : nullptr;
  p.value_cache = app ? const_cast<void*>(value_cache) : nullptr;
  p.slot_out = app ? app->slot_out : nullptr;
  auto st = (cudaStream_t)stream;
  if (prefix && !kv_fp8 && head_dim == 128) {
    // shared prefix: whole partitions inside it, batched across sequences
    // when a CTA's 16 query columns hold at least two sequences
    const int n_prefix = (prefix->len / block_size) / p.part_blocks;
    p.seq_group = 16 / group;
    if (n_prefix > 0 && p.seq_group >= 2) {
      p.prefix_blocks = prefix->blocks;
      if (dtype == PA_BF16) {
        if (block_size == 16)
          return run_shared_prefix<__nv_bfloat16, 16>(mk, mv, p, num_parts, n_prefix, st);
        return run_shared_prefix<__nv_bfloat16, 32>(mk, mv, p, num_parts, n_prefix, st);
      }
      if (block_size == 16) return run_shared_prefix<__half, 16>(mk, mv, p, num_parts, n_prefix, st);
      return run_shared_prefix<__half, 32>(mk, mv, p, num_parts, n_prefix, st);
    }
    p.seq_group = 1;  // otherwise: plain pa_decode
  }
  if (kv_fp8) {
    if (dtype == PA_BF16) return dispatch_decode_fp8<__nv_bfloat16>(block_size, mk, mv, p, num_parts, st);
    return dispatch_decode_fp8<__half>(block_size, mk, mv, p, num_parts, st);
  }
  if (dtype == PA_BF16)
    return dispatch_decode<__nv_bfloat16>(head_dim, block_size, mk, mv, p, num_parts, st);
  return dispatch_decode<__half>(head_dim, block_size, mk, mv, p, num_parts, st);
}

}  // namespace

extern "C" {

pa_status pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, int max_seq_len,
                    int partition_tokens, float scale, pa_dtype dtype, void* workspace,
                    size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, seq_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_blocks_per_seq, max_seq_len, partition_tokens, scale, 1.f, 1.f, false,
                     dtype, workspace, workspace_bytes, stream);
}

pa_status pa_append_decode(void* out, const void* query, const void* new_key,
                           const void* new_value, void* key_cache, void* value_cache,
                           const int32_t* block_tables, const int32_t* ctx_lens,
                           int64_t* slot_mapping, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, int max_ctx_len, int partition_tokens,
                           float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                           pa_stream_t stream) {
  if (max_ctx_len < 0 || max_ctx_len == INT_MAX) return PA_ERR_INVALID_ARG;  // decodes ctx + 1
  const AppendArgs app{new_key, new_value, slot_mapping};
  return decode_impl(out, query, key_cache, value_cache, block_tables, ctx_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_blocks_per_seq, max_ctx_len + 1, partition_tokens, scale, 1.f, 1.f,
                     false, dtype, workspace, workspace_bytes, stream, &app);
}

pa_status pa_decode_shared_prefix(void* out, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* prefix_blocks,
                                  int prefix_len, const int32_t* block_tables,
                                  const int32_t* seq_lens, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  int max_blocks_per_seq, int max_seq_len, int partition_tokens,
                                  float scale, pa_dtype dtype, void* workspace,
                                  size_t workspace_bytes, pa_stream_t stream) {
  const PrefixArgs prefix{prefix_blocks, prefix_len};
  return decode_impl(out, query, key_cache, value_cache, block_tables, seq_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_blocks_per_seq, max_seq_len, partition_tokens, scale, 1.f, 1.f, false,
                     dtype, workspace, workspace_bytes, stream, nullptr, &prefix);
}

pa_status pa_append_decode_fp8(void* out, const void* query, const void* new_key,
                               const void* new_value, uint8_t* key_cache, uint8_t* value_cache,
                               const int32_t* block_tables, const int32_t* ctx_lens,
                               int64_t* slot_mapping, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               int max_blocks_per_seq, int max_ctx_len, int partition_tokens,
                               float scale, float k_scale, float v_scale, pa_dtype dtype,
                               void* workspace, size_t workspace_bytes, pa_stream_t stream) {
  if (max_ctx_len < 0 || max_ctx_len == INT_MAX) return PA_ERR_INVALID_ARG;  // decodes ctx + 1
  const AppendArgs app{new_key, new_value, slot_mapping};
  return decode_impl(out, query, key_cache, value_cache, block_tables, ctx_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_blocks_per_seq, max_ctx_len + 1, partition_tokens, scale, k_scale,
                     v_scale, true, dtype, workspace, workspace_bytes, stream, &app);
}

pa_status pa_decode_fp8(void* out, const void* query, const uint8_t* key_cache,
                        const uint8_t* value_cache, const int32_t* block_tables,
                        const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                        int max_seq_len, int partition_tokens, float scale, float k_scale,
                        float v_scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                        pa_stream_t stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, seq_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_blocks_per_seq, max_seq_len, partition_tokens, scale, k_scale, v_scale,
                     true, dtype, workspace, workspace_bytes, stream);
}

pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, uint8_t* key_cache,
                                   uint8_t* value_cache, const int64_t* slot_mapping,
                                   int num_tokens, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, float k_scale, float v_scale,
                                   pa_dtype dtype, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_dtype(dtype) || !std::isfinite(k_scale) || k_scale <= 0.f ||
      !std::isfinite(v_scale) || v_scale <= 0.f)
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if (head_dim % 16 != 0) return PA_ERR_UNSUPPORTED;
  const long long total = (long long)num_tokens * num_kv_heads * (head_dim / 16);
  const int threads = 256;
  const long long grid = (total + threads - 1) / threads;
  if (grid > INT_MAX) return PA_ERR_INVALID_ARG;
  const int64_t num_slots = (int64_t)num_blocks * block_size;
  auto st = (cudaStream_t)stream;
  if (dtype == PA_BF16)
    pa::reshape_and_cache_fp8_kernel<__nv_bfloat16><<<(unsigned)grid, threads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(key), reinterpret_cast<const __nv_bfloat16*>(value),
        key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
        num_slots, k_scale, v_scale);
  else
    pa::reshape_and_cache_fp8_kernel<__half><<<(unsigned)grid, threads, 0, st>>>(
        reinterpret_cast<const __half*>(key), reinterpret_cast<const __half*>(value), key_cache,
        value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size, num_slots,
        k_scale, v_scale);
  return launch_status();
}

pa_status pa_decode_static_workspace(void* out, const void* query, const void* key_cache,
                                     const void* value_cache, const int32_t* block_tables,
                                     const int32_t* seq_lens, int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int max_blocks_per_seq, int max_seq_len,
                                     int partition_tokens, float scale, pa_dtype dtype,
                                     pa_stream_t stream) {
  size_t need = 0;
  pa_status st = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                          block_size, max_seq_len, partition_tokens, &need);
  if (st != PA_OK) return st;
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    st = static_workspace_address(&ws);
    if (st != PA_OK) return st;
  }
  return pa_decode(out, query, key_cache, value_cache, block_tables, seq_lens, num_seqs,
                   num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                   max_blocks_per_seq, max_seq_len, partition_tokens, scale, dtype, ws,
                   need > 0 ? (size_t)PA_STATIC_WORKSPACE_BYTES : 0, stream);
}

pa_status pa_prefill_workspace_size(int head_dim, size_t* bytes) {
  if (!bytes || head_dim <= 0) return PA_ERR_INVALID_ARG;
  *bytes = prefill_workspace_bytes(head_dim);
  return PA_OK;
}

pa_status pa_prefill_chunk(void* out, const void* query, const void* key_cache,
                           const void* value_cache, const int32_t* block_tables,
                           const int32_t* cu_q_lens, const int32_t* ctx_lens, int num_seqs,
                           int total_q, int max_q_len, int max_ctx_len, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_blocks_per_seq, float scale, pa_dtype dtype, void* workspace,
                           size_t workspace_bytes, pa_stream_t stream) {
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || max_ctx_len < 0 || num_q_heads <= 0 ||
      num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || !valid_dtype(dtype) ||
      !std::isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !cu_q_lens || !ctx_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  if ((long long)max_ctx_len >= (long long)max_blocks_per_seq * block_size)
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 65535 || num_q_heads > 65535) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if ((long long)num_blocks * num_kv_heads * block_size > INT_MAX) return PA_ERR_INVALID_ARG;
  if ((long long)total_q * num_q_heads * head_dim > INT_MAX) return PA_ERR_INVALID_ARG;

  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)num_blocks * num_kv_heads * block_size;
  if (!make_map_2d(&mq, query, (uint64_t)num_q_heads * head_dim, total_q,
                   (uint64_t)num_q_heads * head_dim, 128, dtype) ||
      !make_map_2d(&mk, key_cache, head_dim, rows, head_dim, block_size, dtype) ||
      !make_map_2d(&mv, value_cache, head_dim, rows, head_dim, block_size, dtype))
    return PA_ERR_CUDA;
  pa::PrefillParams p;
  p.out = out;
  p.block_tables = block_tables;
  p.cu_q_lens = cu_q_lens;
  p.ctx_lens = ctx_lens;
  p.num_seqs = num_seqs;
  p.total_q = total_q;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.num_blocks = num_blocks;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.tiles_per_seq = (max_q_len + 255) / 256;
  const bool have_ws = workspace != nullptr && workspace_bytes >= prefill_workspace_bytes(head_dim);
  plan_prefill_split(p, (long long)p.tiles_per_seq * num_q_heads * num_seqs, have_ws);
  if (p.split > 1) {
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
    p.counters = reinterpret_cast<int*>(base);
    p.ws_o = reinterpret_cast<float*>(base + kPrefillCounterBytes);
    p.ws_ml = p.ws_o + (size_t)kPrefillPartWaves * sm_count() * 256 * head_dim;
  } else {
    p.counters = nullptr;
    p.ws_o = p.ws_ml = nullptr;
  }
  return dispatch_prefill(mq, mk, mv, p, dtype, block_size, head_dim, (cudaStream_t)stream);
}

pa_status pa_mixed_workspace_size(int num_decode_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int block_size, int max_ctx_len,
                                  int partition_tokens, size_t* bytes) {
  if (!bytes || num_decode_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_ctx_len < 0 || max_ctx_len == INT_MAX || partition_tokens < 0)
    return PA_ERR_INVALID_ARG;
  const int max_dec_len = max_ctx_len + 1;
  const int pt = mixed_partition_tokens(partition_tokens, num_decode_seqs > 0 ? num_decode_seqs : 1,
                                        num_kv_heads, block_size, max_dec_len);
  // pt >= 1, so the count fits an int
  *bytes = mixed_workspace_bytes(num_decode_seqs, num_q_heads, head_dim,
                                 (int)num_partitions(max_dec_len, pt));
  return PA_OK;
}

pa_status pa_mixed_attention(void* out, const void* query, const void* key_cache,
                             const void* value_cache, const int32_t* block_tables,
                             const int32_t* cu_q_lens, const int32_t* ctx_lens, int num_seqs,
                             int num_decode_seqs, int total_q, int max_q_len, int max_ctx_len,
                             int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int max_blocks_per_seq, int partition_tokens,
                             float scale, pa_dtype dtype, void* workspace,
                             size_t workspace_bytes, pa_stream_t stream) {
  if (num_seqs < 0 || num_decode_seqs < 0 || num_decode_seqs > num_seqs ||
      total_q < num_decode_seqs || max_q_len < 0 || max_ctx_len < 0 || max_ctx_len == INT_MAX ||
      num_q_heads <= 0 ||
      num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || partition_tokens < 0 ||
      !valid_dtype(dtype) || !std::isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || total_q == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !cu_q_lens || !ctx_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_INVALID_ARG;
  // a decode row attends over ctx + 1 tokens, which must fit the table
  if ((long long)max_ctx_len >= (long long)max_blocks_per_seq * block_size)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads > 65535) return PA_ERR_INVALID_ARG;
  if (head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if ((long long)num_blocks * num_kv_heads * block_size > INT_MAX) return PA_ERR_INVALID_ARG;
  if ((long long)total_q * num_q_heads * head_dim > INT_MAX) return PA_ERR_INVALID_ARG;

  // decode rows: split-KV plan over lengths up to max_ctx_len + 1
  const int num_decode = num_decode_seqs;
  const int max_dec_len = max_ctx_len + 1;
  const int pt = mixed_partition_tokens(partition_tokens, num_decode > 0 ? num_decode : 1,
                                        num_kv_heads, block_size, max_dec_len);
  const int num_parts = (int)num_partitions(max_dec_len, pt);
  const size_t need = mixed_workspace_bytes(num_decode, num_q_heads, head_dim, num_parts);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return PA_ERR_WORKSPACE;
  // prefill chunks: 256-row tiles per (chunk, query head)
  const int num_prefill = num_seqs - num_decode;
  const long long tiles = (num_prefill > 0 && max_q_len > 0) ? (max_q_len + 255) / 256 : 0;
  const long long prefill_ctas = tiles * num_q_heads * num_prefill;
  const long long decode_items = (long long)num_decode * num_kv_heads * num_parts;
  if (prefill_ctas >= INT_MAX || decode_items > INT_MAX) return PA_ERR_INVALID_ARG;

  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)num_blocks * num_kv_heads * block_size;
  if (!make_map_2d(&mq, query, (uint64_t)num_q_heads * head_dim, total_q,
                   (uint64_t)num_q_heads * head_dim, 128, dtype) ||
      !make_map_2d(&mk, key_cache, head_dim, rows, head_dim, block_size, dtype) ||
      !make_map_2d(&mv, value_cache, head_dim, rows, head_dim, block_size, dtype))
    return PA_ERR_CUDA;

  pa::PrefillParams pp;
  pp.out = out;
  pp.block_tables = block_tables;
  pp.cu_q_lens = cu_q_lens;
  pp.ctx_lens = ctx_lens;
  pp.num_seqs = num_seqs;
  pp.total_q = total_q;
  pp.num_q_heads = num_q_heads;
  pp.num_kv_heads = num_kv_heads;
  pp.group = group;
  pp.num_blocks = num_blocks;
  pp.max_blocks_per_seq = max_blocks_per_seq;
  pp.scale_log2 = scale * 1.4426950408889634f;
  pp.tiles_per_seq = (int)(tiles > 0 ? tiles : 1);
  pp.n_full = (int)prefill_ctas;
  pp.split = 1;
  pp.ws_o = pp.ws_ml = nullptr;
  pp.counters = nullptr;

  pa::DecodeParams dp;
  dp.out = out;
  dp.query = query;
  dp.block_tables = block_tables;
  dp.seq_lens = ctx_lens;
  dp.len_add = 1;
  dp.new_key = dp.new_value = nullptr;
  dp.key_cache = dp.value_cache = nullptr;
  dp.slot_out = nullptr;
  uint8_t* ws_base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  float* ws = reinterpret_cast<float*>(ws_base + 256);
  const size_t acc_elems = (size_t)num_decode * num_q_heads * num_parts * head_dim;
  dp.ws_acc = num_parts > 1 && need > 0 ? ws : nullptr;
  dp.ws_ml = num_parts > 1 && need > 0 ? ws + acc_elems : nullptr;
  dp.num_seqs = num_decode;
  dp.num_q_heads = num_q_heads;
  dp.num_kv_heads = num_kv_heads;
  dp.group = group;
  dp.num_blocks = num_blocks;
  dp.max_blocks_per_seq = max_blocks_per_seq;
  dp.part_blocks = pt / block_size;
  dp.max_parts = num_parts;
  dp.scale_log2 = pp.scale_log2;
  dp.v_scale = 1.f;

  pa::MixedPlan plan;
  plan.prefill_ctas = (int)prefill_ctas;
  plan.prefill_slots = (int)((prefill_ctas + 1) & ~1LL);
  plan.prefill_tiles = (int)(tiles > 0 ? tiles : 1);
  plan.first_prefill_seq = num_decode;
  plan.decode_items = (int)decode_items;
  plan.queue = need > 0 ? reinterpret_cast<int*>(ws_base) : nullptr;

  auto st = (cudaStream_t)stream;
  if (plan.queue != nullptr && cudaMemsetAsync(plan.queue, 0, sizeof(int), st) != cudaSuccess)
    return PA_ERR_CUDA;
  if (dtype == PA_BF16) {
    if (block_size == 16)
      return dispatch_mixed<__nv_bfloat16, 16>(group, mq, mk, mv, pp, dp, plan, st);
    return dispatch_mixed<__nv_bfloat16, 32>(group, mq, mk, mv, pp, dp, plan, st);
  }
  if (block_size == 16) return dispatch_mixed<__half, 16>(group, mq, mk, mv, pp, dp, plan, st);
  return dispatch_mixed<__half, 32>(group, mq, mk, mv, pp, dp, plan, st);
}

pa_status pa_selftest_wait_timeout(uint64_t limit_ns, uint64_t* waited_ns, pa_stream_t stream) {
  if (limit_ns < 1000ull || limit_ns > 100000000ull) return PA_ERR_INVALID_ARG;
  if (waited_ns != nullptr && (reinterpret_cast<uintptr_t>(waited_ns) & 7u) != 0)
    return PA_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(limit_ns, waited_ns);
  return launch_status();
}

pa_status pa_get_device_error(unsigned int* error_word, pa_stream_t stream) {
  if (!error_word) return PA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_error_word, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return PA_ERR_CUDA;
  *error_word = v;
  return v == 0 ? PA_OK : PA_ERR_OUT_OF_RANGE;
}

}  // extern "C"
