// C-ABI entry points of the attention library (declared in include/attn.h).
//
// This file is the only translation unit: it includes every kernel, so the
// device status word has exactly one definition. Host work per call is
// argument validation, tensor-map encoding (three to five 3-D maps) and the
// kernel launches; nothing is allocated and nothing is synchronised except in
// attn_check_status().
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <memory>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "../../include/attn.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "sm100.cuh"

namespace {

thread_local char g_last_error[512] = "";

attn_status fail(attn_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

attn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ATTN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---------------------------------------------------------------- profiling
// Opt-in per-kernel timing: when enabled, every launch is bracketed by two
// CUDA events recorded on the launch stream; attn_profile_read() sums the
// elapsed times per kernel. Events come from a pool that grows on demand.
enum ProfKernel { kProfFwd = 0, kProfBwdPre, kProfBwdDkdv, kProfBwdDq, kProfCount };
const char* const kProfNames[kProfCount] = {"fwd_kernel", "bwd_pre_kernel", "bwd_dkdv_kernel",
                                            "bwd_dq_kernel"};

struct ProfState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  struct Pending { int kernel; cudaEvent_t a, b; };
  std::vector<Pending> pending;
  int launches[kProfCount] = {0, 0, 0, 0};
  double total_ms[kProfCount] = {0, 0, 0, 0};
};
ProfState g_prof;

cudaEvent_t prof_event() {
  if (!g_prof.pool.empty()) {
    cudaEvent_t e = g_prof.pool.back();
    g_prof.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch when profiling is on. Usage: ProfScope ps(kernel, s); launch; ps.end();
struct ProfScope {
  int kernel;
  cudaStream_t stream;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(int k, cudaStream_t s) : kernel(k), stream(s) {
    std::lock_guard<std::mutex> g(g_prof.mu);
    if (!g_prof.on) return;
    a = prof_event();
    b = prof_event();
    if (a && b) cudaEventRecord(a, stream);
  }
  void end() {
    if (!a || !b) return;
    cudaEventRecord(b, stream);
    std::lock_guard<std::mutex> g(g_prof.mu);
    g_prof.pending.push_back({kernel, a, b});
  }
};

// ---------------------------------------------------------------- driver entry
// cuTensorMapEncodeTiled is a driver API call; it is fetched through the
// runtime so the library links only the static CUDA runtime and can be
// loaded (for symbol checks) on a machine without a GPU driver.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;
attn_status g_init_status = ATTN_OK;
char g_init_msg[256] = "";
std::once_flag g_init_once;

// Devices a process may use (per-device caches below are indexed by ordinal).
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};             // multiprocessors, filled by check_device()

// The device current for the API call this thread is in. check_device(),
// which every entry point runs before anything that needs the device, sets
// it, so the rest of the call does not query the runtime again.
thread_local int t_call_dev = -1;

int call_device() {
  if (t_call_dev >= 0) return t_call_dev;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int sm_count() {
  const int dev = call_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  return g_sm_count[dev] > 0 ? g_sm_count[dev] : 148;
}

void init_once() {
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) {
    g_init_status = ATTN_ERR_CUDA;
    snprintf(g_init_msg, sizeof(g_init_msg), "cuTensorMapEncodeTiled unavailable (%s)",
             cudaGetErrorString(e));
    return;
  }
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}

// The current device must be an sm_100 part; checked once per device.
attn_status check_device() {
  t_call_dev = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ATTN_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(ATTN_ERR_CUDA, "device index %d unsupported", dev);
  // 0: not checked yet, else major * 10 + minor. Written once per device
  // under the mutex (after g_sm_count), read without it afterwards.
  static std::mutex mu;
  static std::atomic<int> arch[kMaxDevices] = {};
  int a = arch[dev].load(std::memory_order_acquire);
  if (a == 0) {
    std::lock_guard<std::mutex> g(mu);
    a = arch[dev].load(std::memory_order_relaxed);
    if (a == 0) {
      cudaDeviceProp prop;
      e = cudaGetDeviceProperties(&prop, dev);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(ATTN_ERR_CUDA, "cudaGetDeviceProperties(%d): %s", dev,
                    cudaGetErrorString(e));
      }
      g_sm_count[dev] = prop.multiProcessorCount;
      a = prop.major * 10 + prop.minor;
      arch[dev].store(a, std::memory_order_release);
    }
  }
  if (a != 100)
    return fail(ATTN_ERR_CUDA, "this library is built for sm_100a (B200); device %d is sm_%d", dev,
                a);
  t_call_dev = dev;
  return ATTN_OK;
}

attn_status ensure_init() {
  attn_status st = check_device();
  if (st != ATTN_OK) return st;
  std::call_once(g_init_once, init_once);
  if (g_init_status != ATTN_OK) return fail(g_init_status, "%s", g_init_msg);
  return ATTN_OK;
}

// One-time setup of a kernel on each device it runs on: the dynamic shared
// memory opt-in applies to the device current when it is made. Also records
// the register count ptxas gave the kernel (the forward checks it against its
// setmaxnreg split).
struct KernelSetup {
  std::mutex mu;
  std::atomic<bool> done[kMaxDevices] = {};   // set (release) after err and regs
  cudaError_t err[kMaxDevices] = {};
  int regs[kMaxDevices] = {};
};

template <typename Kern>
cudaError_t prepare_kernel(Kern kern, int smem_bytes, KernelSetup& ks, int* regs = nullptr) {
  const int dev = call_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!ks.done[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> g(ks.mu);
    if (!ks.done[dev].load(std::memory_order_relaxed)) {
      cudaError_t e =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
      cudaFuncAttributes fa;
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
      ks.err[dev] = e;
      ks.regs[dev] = (e == cudaSuccess) ? fa.numRegs : 0;
      ks.done[dev].store(true, std::memory_order_release);
    }
  }
  if (regs) *regs = ks.regs[dev];
  return ks.err[dev];
}
// Launch with programmatic stream serialization: the kernel may be launched
// while the kernel before it on the stream finishes (every kernel here waits
// for its predecessor with griddepcontrol.wait before touching global memory,
// and allows its successor's launch once all its CTAs have finished their
// work). Between two launches of this library that hides the launch latency
// and the next kernel's set-up, which is what short problems are made of.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, int threads, int smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// 3-D tensor map (d, rows, z) over a bf16 tensor, with a box of 64 x 128 x 1
// (one 128-row, 128-byte-wide column block) and 128-byte swizzle. Row and z
// strides are in elements. Fixed-length [B*H, N, d]: rows = N, z = B*H,
// row stride d, z stride N*d. Packed [total, H, d]: rows = total, z = H, row
// stride H*d, z stride d. Rows past `rows` read as zeros, and stores to them
// are dropped.
// Recently encoded maps, per calling thread: training and serving loops call
// with the same tensors again and again, and an encode costs about as much
// host time as the launch. A map depends only on these arguments (it holds
// the global address, extents and strides, nothing device-specific).
struct MapKey {
  const void* base;
  long long rows, zdim, row_stride, z_stride;
  int d;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && zdim == o.zdim && row_stride == o.row_stride &&
           z_stride == o.z_stride && d == o.d;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kMapCacheSize = 16;
thread_local MapEntry t_map_cache[kMapCacheSize] = {};
thread_local int t_map_next = 0;

attn_status make_map(CUtensorMap* map, const void* base, int d, long long rows, long long zdim,
                     long long row_stride, long long z_stride) {
  const MapKey key{base, rows, zdim, row_stride, z_stride, d};
  for (int i = 0; i < kMapCacheSize; ++i)
    if (t_map_cache[i].valid && t_map_cache[i].key == key) {
      *map = t_map_cache[i].map;
      return ATTN_OK;
    }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(zdim)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride) * 2,
                           static_cast<cuuint64_t>(z_stride) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  MapEntry& e = t_map_cache[t_map_next];
  t_map_next = (t_map_next + 1) % kMapCacheSize;
  e.key = key;
  e.map = *map;
  e.valid = true;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Null, alignment, memory-kind and device checks for the tensor arguments. A
// host pointer, or memory of another GPU than the current one, handed to a
// kernel would fault the GPU, so both are rejected here.
attn_status check_device_ptr(const void* ptr, const char* name) {
  const int dev = call_device();
  if (dev < 0) return fail(ATTN_ERR_CUDA, "cudaGetDevice failed");
  cudaPointerAttributes pa;
  cudaError_t e = cudaPointerGetAttributes(&pa, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ATTN_ERR_ARG, "%s is not a CUDA pointer (%s)", name, cudaGetErrorName(e));
  }
  if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)
    return fail(ATTN_ERR_ARG, "%s is not device memory", name);
  if (pa.type == cudaMemoryTypeDevice && pa.device != dev)
    return fail(ATTN_ERR_ARG, "%s lives on device %d but the current device is %d", name,
                pa.device, dev);
  return ATTN_OK;
}

attn_status check_ptrs(const void* const* ptrs, const char* const* names, int n) {
  for (int i = 0; i < n; ++i) {
    if (ptrs[i] == nullptr) return fail(ATTN_ERR_ARG, "%s is null", names[i]);
    if (!aligned16(ptrs[i])) return fail(ATTN_ERR_ARG, "%s is not 16-byte aligned", names[i]);
  }
  for (int i = 0; i < n; ++i) {
    attn_status st = check_device_ptr(ptrs[i], names[i]);
    if (st != ATTN_OK) return st;
  }
  return ATTN_OK;
}

// Shape checks shared by forward and backward. Returns ATTN_OK and sets
// *empty when there is nothing to compute.
attn_status check_shape(int B, int Hq, int Hkv, int N, int d, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || N < 0) return fail(ATTN_ERR_ARG, "B and N must be >= 0 (got B=%d N=%d)", B, N);
  if (Hq < 1 || Hkv < 1) return fail(ATTN_ERR_ARG, "Hq and Hkv must be >= 1 (got %d, %d)", Hq, Hkv);
  if (Hq % Hkv != 0)
    return fail(ATTN_ERR_ARG, "Hq (%d) must be divisible by Hkv (%d) for MQA/GQA", Hq, Hkv);
  if (d != 64 && d != 128)
    return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not supported (built: 64, 128)", d);
  if (!(scale > 0.f) || !std::isfinite(scale))
    return fail(ATTN_ERR_ARG, "scale must be finite and > 0 (got %g)", (double)scale);
  if (static_cast<long long>(B) * Hq > 0x7FFFFFFFLL)
    return fail(ATTN_ERR_ARG, "B*Hq too large");
  if (N > (1 << 24)) return fail(ATTN_ERR_ARG, "N=%d exceeds the supported maximum 2^24", N);
  if (B == 0 || N == 0) *empty = true;
  return ATTN_OK;
}

// Which keys each query row sees: the three kernel mask modes and the window
// bounds they use. window_left/right < 0 is unbounded; causal caps the right
// side at 0. Same-length problems without a left window keep the unmasked
// and causal fast paths. Packed batches and softcapping always run the
// general mode (its bounds are per sequence; the softcap variant exists only
// there). The kernels set the offset Nk - Nq per sequence.
struct MaskSpec {
  int mode;
  bool softcap;
  attn::KeyWindow win;
};

MaskSpec mask_spec(int Nq, int Nk, int causal, int window_left, int window_right, bool packed,
                   float softcap) {
  using namespace attn;
  const int wl = window_left < 0 ? kUnbounded : std::min(window_left, kUnbounded);
  int wr = window_right < 0 ? kUnbounded : std::min(window_right, kUnbounded);
  if (causal) wr = 0;
  const bool plain = !packed && softcap == 0.f && Nq == Nk && wl == kUnbounded &&
                     (causal || wr == kUnbounded);
  const int mode = plain ? (causal ? kMaskCausal : kMaskNone) : kMaskGeneral;
  return MaskSpec{mode, softcap > 0.f, KeyWindow{Nk - Nq, wl, wr}};
}

// Everything a launch needs besides the tensor maps.
struct Problem {
  int B, Hq, Hkv, d;
  attn::SeqGeom geom;
  float scale;
  MaskSpec mask;
  attn::Softcap cap;
};

// Heads per group of the forward's grid order (the list is walked group by
// group, heaviest block first within a group).
// - Unmasked: consecutive (batch, query head) indices whose K and V together
//   stay well inside L2 (about 48 MB of the 126 MB), rounded down to whole GQA
//   groups. Measured on B200 (c3, N 4096 d 128): 1076 -> 1137-1155 TFLOP/s.
// - Causal: the smallest group whose block count is a whole number of snake
//   periods (2 x grid entries), so the heavy-to-light order of each group
//   balances the CTAs by itself, if its K and V fit in 80 MB; else one group.
//   An L2-sized group that broke the periods was slower (c3 1012 -> 913); the
//   aligned one is faster (c3 1021 -> 1044, c5 851 -> 861 TFLOP/s).
// - Other masks (windows): one group.
// A causal problem that runs with a plan (below) uses the plan's group size.
int fwd_head_group(const Problem& p, int nmb, int grid) {
  const long long all = static_cast<long long>(p.B) * p.Hq;
  if (p.mask.mode == attn::kMaskCausal) {
    long long a = 2LL * grid, b = nmb;     // a = gcd(2 grid, nmb) after the loop
    while (b) {
      const long long t = a % b;
      a = b;
      b = t;
    }
    const long long hg = 2LL * grid / a;   // >= 1, and hg * nmb is a multiple of 2 grid
    const double kv_bytes_per_head = 2.0 * p.geom.Nk * p.d * 2.0 / (p.Hq / p.Hkv);
    if (hg < all && hg * kv_bytes_per_head <= 80.0 * (1 << 20)) return static_cast<int>(hg);
    return static_cast<int>(all);
  }
  if (p.mask.mode != attn::kMaskNone) return static_cast<int>(all);
  const int group = p.Hq / p.Hkv;
  const double kv_bytes_per_head = 2.0 * p.geom.Nk * p.d * 2.0 / group;
  const double budget = 48.0 * (1 << 20);
  long long hg = static_cast<long long>(budget / std::max(kv_bytes_per_head, 1.0));
  hg = std::max<long long>(group, hg - hg % group);
  return static_cast<int>(std::min<long long>(hg, all));
}

// ---------------------------------------------------------------- causal plan
// Causal blocks differ in cost: block mb of a head has about 2 mb + 2 key-tile
// steps. When the block count is not a whole number of snake periods, the
// snake leaves some CTAs with much more work than others (c5, 1024 blocks on
// 148 CTAs: 54 to 70 steps, 62.3 on average). The plan instead hands each list
// entry, in list order, to the CTA with the least work so far, costed as its
// key-tile steps plus kPlanBlockCost steps for the block's start and end (clock
// stamps: a 256-row block pays about 2.5 us at its boundary, a step about 1.9
// us). It keeps the list order, so heads still come in groups that fit L2.

constexpr double kPlanBlockCost = 1.3;

// The list entries' costs for a causal fixed-length problem, in list order
// (the same decoding as fwd_block).
std::vector<double> causal_costs(const attn::FwdSched& sc, int N) {
  std::vector<double> cost(static_cast<size_t>(sc.total));
  const int rb = sc.one_tile ? 128 : 256;
  const long long per_group = static_cast<long long>(sc.hg) * sc.nmb;
  for (long long idx = 0; idx < sc.total; ++idx) {
    const long long g = idx / per_group, r = idx - g * per_group;
    const long long gs = std::min<long long>(sc.hg, sc.BH - g * sc.hg);
    const int mb = sc.nmb - 1 - static_cast<int>(r / gs);
    const int m0 = mb * rb;
    int lo = 0, hi = -1;
    attn::kv_tile_range<attn::kMaskCausal>(m0, std::min(m0 + rb - 1, N - 1), N, attn::KeyWindow{},
                                           lo, hi);
    cost[static_cast<size_t>(idx)] = (hi - lo + 1) + kPlanBlockCost;
  }
  return cost;
}

// Largest per-CTA cost of the snake assignment.
double snake_makespan(const std::vector<double>& cost, int grid) {
  std::vector<double> load(static_cast<size_t>(grid), 0.0);
  for (size_t idx = 0; idx < cost.size(); ++idx) {
    const size_t t = idx / grid, c = idx % grid;
    load[(t & 1) ? grid - 1 - c : c] += cost[idx];
  }
  return *std::max_element(load.begin(), load.end());
}

// List scheduling in list order onto the least-loaded CTA (lowest index on
// ties). Fills `owner` and returns the largest per-CTA cost.
double list_schedule(const std::vector<double>& cost, int grid, std::vector<int>* owner) {
  using Slot = std::pair<double, int>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int c = 0; c < grid; ++c) heap.push({0.0, c});
  double makespan = 0.0;
  if (owner) owner->resize(cost.size());
  for (size_t idx = 0; idx < cost.size(); ++idx) {
    Slot sl = heap.top();
    heap.pop();
    sl.first += cost[idx];
    makespan = std::max(makespan, sl.first);
    if (owner) (*owner)[idx] = sl.second;
    heap.push(sl);
  }
  return makespan;
}

struct PlanKey {
  long long total;
  int BH, nmb, one_tile, N, grid, group;
  double kv_head;
  bool operator==(const PlanKey& o) const {
    return total == o.total && BH == o.BH && nmb == o.nmb && one_tile == o.one_tile &&
           N == o.N && grid == o.grid && group == o.group && kv_head == o.kv_head;
  }
};
struct PlanEntry {
  PlanKey key;
  std::shared_ptr<const attn::FwdPlan> plan;   // null: the snake is as good
  int hg;
};
std::mutex g_plan_mu;
std::vector<PlanEntry> g_plans;                // a few recent shapes, newest last

// The plan for a causal fixed-length problem, or null when the snake is within
// 2 % of it. Head groups: the sizes that divide the heads evenly (whole GQA
// groups) with K and V of at most 48 MB, the one with the smallest planned
// makespan. Sets sc->hg to the group size the returned plan (or the snake)
// uses. Cached per shape.
std::shared_ptr<const attn::FwdPlan> causal_plan(const Problem& p, int grid, attn::FwdSched* sc) {
  const int group = p.Hq / p.Hkv;
  const double kv_head = 2.0 * p.geom.Nk * p.d * 2.0 / group;
  const PlanKey key{sc->total, sc->BH, sc->nmb, sc->one_tile, p.geom.Nq, grid, group, kv_head};
  {
    std::lock_guard<std::mutex> g(g_plan_mu);
    for (const PlanEntry& e : g_plans)
      if (e.key == key) {
        sc->hg = e.hg;
        return e.plan;
      }
  }
  const double snake = snake_makespan(causal_costs(*sc, p.geom.Nq), grid);
  const int snake_hg = sc->hg;
  int best_hg = 0;
  double best = 0.0;
  for (int hg = group; hg <= sc->BH; hg += group) {
    if (sc->BH % hg != 0 || (hg > group && hg * kv_head > 48.0 * (1 << 20))) continue;
    sc->hg = hg;
    const double m = list_schedule(causal_costs(*sc, p.geom.Nq), grid, nullptr);
    if (best_hg == 0 || m < best * 0.999) {
      best = m;
      best_hg = hg;
    }
  }
  std::shared_ptr<attn::FwdPlan> plan;
  if (best_hg > 0 && best < 0.98 * snake) {
    sc->hg = best_hg;
    std::vector<int> owner;
    list_schedule(causal_costs(*sc, p.geom.Nq), grid, &owner);
    plan = std::make_shared<attn::FwdPlan>();
    std::vector<int> count(static_cast<size_t>(grid) + 1, 0);
    for (int c : owner) ++count[static_cast<size_t>(c) + 1];
    plan->start[0] = 0;
    for (int c = 0; c < grid; ++c)
      plan->start[c + 1] = static_cast<uint16_t>(plan->start[c] + count[static_cast<size_t>(c) + 1]);
    std::vector<int> fill(plan->start, plan->start + grid);
    for (size_t idx = 0; idx < owner.size(); ++idx)
      plan->item[fill[static_cast<size_t>(owner[idx])]++] = static_cast<uint16_t>(idx);
  } else {
    sc->hg = snake_hg;
  }
  std::lock_guard<std::mutex> g(g_plan_mu);
  if (g_plans.size() >= 8) g_plans.erase(g_plans.begin());
  g_plans.push_back(PlanEntry{key, plan, sc->hg});
  return plan;
}

template <int D, int MODE, int FEAT, bool PLAN, bool DB>
attn_status launch_fwd_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mo, void* o, float* lse, const Problem& p,
                              const attn::FwdSched& sched, dim3 grid,
                              const typename attn::FwdPlanArg<PLAN>::type& plan,
                              cudaStream_t stream) {
  using Cfg = attn::FwdCfg<D>;
  auto kern = attn::fwd_kernel<D, MODE, FEAT, PLAN, DB>;
  static KernelSetup setup;
  int launch_regs = 0;
  const cudaError_t attr_err = prepare_kernel(kern, Cfg::kSmemAlloc, setup, &launch_regs);
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(fwd)");
  // The kernel rebalances registers between warpgroups with setmaxnreg; that
  // split is only valid for the launch register count it was written for.
  if (launch_regs != attn::kFwdRegsLaunch)
    return fail(ATTN_ERR_CUDA, "fwd kernel built with %d registers/thread, expected %d",
                launch_regs, attn::kFwdRegsLaunch);
  const float scale_log2 = p.scale * 1.4426950408889634f;
  ProfScope ps(kProfFwd, stream);
  cudaError_t e = launch_pdl(kern, grid, Cfg::kThreads, Cfg::kSmemAlloc, stream, mq, mk, mv, mo,
                             static_cast<__nv_bfloat16*>(o), lse, p.Hq, p.Hq / p.Hkv, p.geom,
                             scale_log2, p.mask.win, p.cap, sched, plan);
  ps.end();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "fwd kernel launch");
  }
  return ATTN_OK;
}

template <int D, int MODE, int FEAT>
attn_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mo, void* o, float* lse, const Problem& p,
                       cudaStream_t stream) {
  // Work items are 256-row query blocks: two 128-row tiles share each K/V
  // tile. When there are fewer blocks than SMs, 128-row blocks (one tile)
  // double their number. The grid is persistent: one CTA per SM, or one per
  // block when there are fewer blocks.
  attn::FwdSched sched;
  sched.BH = p.B * p.Hq;
  const long long pairs = static_cast<long long>(p.B) * p.Hq * ((p.geom.Nq + 255) / 256);
  sched.one_tile = pairs < sm_count() ? 1 : 0;
  sched.nmb = sched.one_tile ? (p.geom.Nq + 127) / 128 : (p.geom.Nq + 255) / 256;
  sched.total = static_cast<long long>(sched.BH) * sched.nmb;
  const int g = static_cast<int>(std::min<long long>(sched.total, sm_count()));
  sched.hg = fwd_head_group(p, sched.nmb, g);
  if (sched.total > 0x7FFFFFFFLL) return fail(ATTN_ERR_ARG, "problem too large for one launch");
  const dim3 grid(static_cast<unsigned>(g));
  // One-tile blocks double-buffer S in the second tile's tensor memory
  // (2 x 128 S columns + D O columns).
  if (sched.one_tile)
    return launch_fwd_kernel<D, MODE, FEAT, false, true>(mq, mk, mv, mo, o, lse, p, sched, grid,
                                                         attn::FwdNoPlan{0}, stream);
  if constexpr (MODE == attn::kMaskCausal && FEAT == 0) {
    if (sched.total > g && sched.total <= attn::kFwdPlanItems && g <= attn::kFwdPlanCtas) {
      const std::shared_ptr<const attn::FwdPlan> plan = causal_plan(p, g, &sched);
      if (plan)
        return launch_fwd_kernel<D, MODE, FEAT, true, false>(mq, mk, mv, mo, o, lse, p, sched,
                                                             grid, *plan, stream);
    }
  }
  return launch_fwd_kernel<D, MODE, FEAT, false, false>(mq, mk, mv, mo, o, lse, p, sched, grid,
                                                        attn::FwdNoPlan{0}, stream);
}

struct BwdArgs {
  CUtensorMap mq, mk, mv, mdo, mdk, mdv, mdq;
  const void* o;
  const float* lse;
  const void* dO;
  void *dq, *dk, *dv;
  float *L, *Dv;
  int* sched;   // the persistent kernels' work counters (zeroed by the preprocess kernel)
};

template <int D, int MODE, int FEAT>
attn_status launch_bwd(const BwdArgs& a, const Problem& p, cudaStream_t stream) {
  using namespace attn;
  const int Npad = pad128(p.geom.Nq);
  const int group = p.Hq / p.Hkv;
  const float scale_log2 = p.scale * kLog2e;

  const long long rows = static_cast<long long>(p.B) * p.Hq * Npad;
  // dK/dV work items: (batch, KV head, 128-key block); the grid is persistent.
  const long long g1 = static_cast<long long>(pad128(p.geom.Nk) / 128) * p.B * p.Hkv;
  const long long g2 = static_cast<long long>(Npad / 128) * p.B * p.Hq;
  if (rows / 32 > 0x7FFFFFFFLL || g1 > 0x7FFFFFFFLL || g2 > 0x7FFFFFFFLL)
    return fail(ATTN_ERR_ARG, "problem too large for one launch");
  ProfScope p0(kProfBwdPre, stream);
  cudaError_t e = launch_pdl(bwd_pre_kernel<D>, dim3(static_cast<unsigned>(rows / 32)), 256, 0,
                             stream, static_cast<const __nv_bfloat16*>(a.o),
                             static_cast<const __nv_bfloat16*>(a.dO), a.lse, a.L, a.Dv, p.Hq,
                             p.geom, Npad, a.sched);
  p0.end();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "bwd preprocess launch");
  }

  static KernelSetup s1, s2;
  auto k1 = bwd_dkdv_kernel<D, MODE, FEAT>;
  auto k2 = bwd_dq_kernel<D, MODE, FEAT>;
  if ((e = prepare_kernel(k1, DkdvCfg<D>::kSmemAlloc, s1)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(dkdv)");
  if ((e = prepare_kernel(k2, DqCfg<D>::kSmemAlloc, s2)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(dq)");

  ProfScope p1(kProfBwdDkdv, stream);
  const unsigned grid1 = static_cast<unsigned>(std::min<long long>(g1, sm_count()));
  // Heads numbered key-block-major at the end of the item list: enough for
  // two items per CTA, so the lightest blocks of those heads come last.
  const int nkv1 = pad128(p.geom.Nk) / 128;
  const int tail1 = static_cast<int>(std::min<long long>(static_cast<long long>(p.B) * p.Hkv,
                                                         (2LL * grid1 + nkv1 - 1) / nkv1));
  e = launch_pdl(k1, dim3(grid1), DkdvCfg<D>::kThreads, DkdvCfg<D>::kSmemAlloc, stream, a.mq,
                 a.mk, a.mv, a.mdo, a.mdk, a.mdv, a.L, a.Dv, static_cast<__nv_bfloat16*>(a.dk),
                 static_cast<__nv_bfloat16*>(a.dv), p.Hq, group, p.geom, Npad, scale_log2,
                 p.scale, p.mask.win, p.cap, a.sched, static_cast<int>(g1), tail1);
  p1.end();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "bwd dK/dV launch");
  }
  ProfScope p2(kProfBwdDq, stream);
  // dQ work items: (batch, query head, 128-query block); persistent as above.
  const unsigned grid2 = static_cast<unsigned>(std::min<long long>(g2, sm_count()));
  const int nqb2 = Npad / 128;
  const int tail2 = static_cast<int>(std::min<long long>(static_cast<long long>(p.B) * p.Hq,
                                                         (2LL * grid2 + nqb2 - 1) / nqb2));
  e = launch_pdl(k2, dim3(grid2), DqCfg<D>::kThreads, DqCfg<D>::kSmemAlloc, stream, a.mq, a.mk,
                 a.mv, a.mdo, a.mdq, a.L, a.Dv, static_cast<__nv_bfloat16*>(a.dq), p.Hq, group,
                 p.geom, Npad, scale_log2, p.scale, p.mask.win, p.cap, a.sched + 1,
                 static_cast<int>(g2), tail2);
  p2.end();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "bwd dQ launch");
  }
  return ATTN_OK;
}

// ---------------------------------------------------------------- wait self-test
// One thread waits on an mbarrier that nothing ever arrives on, through the
// same bounded wait every pipeline role uses. The wait must give up after
// kWaitTimeoutNs and record a timeout in the status word. This exercises the
// failure-detection path without faulting or hanging the GPU.
__global__ void selftest_wait_timeout_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    attn::mbar_init(&bar, 1);
    abort_flag = 0;
    attn::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) attn::mbar_wait(&bar, 0, &abort_flag, 0x7E);
}

// ---------------------------------------------------------------- static scratch
// Backing store for attn_bwd_noalloc: the backward's lse*log2(e) and
// rowsum(dO*O) rows live in this fixed device array instead of a
// caller-provided workspace. Every device that loads the library holds these
// 8 MiB + 64 bytes until the process exits. Host code must not hand the symbol itself to
// a kernel (on the host it names a stand-in, not device memory). Its device
// address is looked up once per device with cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = (size_t(8) << 20) + attn::kBwdCounterBytes;
static __device__ __align__(256) float g_bwd_scratch[kStaticScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_bwd_scratch on the current device. The first call on
// each device resolves it (with that device current) and caches it.
attn_status static_scratch_ptr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(ATTN_ERR_CUDA, "device index %d unsupported", dev);
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                       "cudaGetSymbolAddress(static backward scratch)");
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return ATTN_OK;
}

// Rows of a problem with no keys: lse = -inf.
__global__ void fill_neg_inf_kernel(float* p, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    p[i] = -INFINITY;
}

template <int D>
attn_status dispatch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo,
                         void* o, float* lse, const Problem& p, cudaStream_t stream) {
  using namespace attn;
  if (p.mask.mode == kMaskNone)
    return launch_fwd<D, kMaskNone, 0>(mq, mk, mv, mo, o, lse, p, stream);
  if (p.mask.mode == kMaskCausal)
    return launch_fwd<D, kMaskCausal, 0>(mq, mk, mv, mo, o, lse, p, stream);
  const bool packed = p.geom.cu_q != nullptr;
  if (packed && p.mask.softcap)
    return launch_fwd<D, kMaskGeneral, kFeatPacked | kFeatSoftcap>(mq, mk, mv, mo, o, lse, p,
                                                                    stream);
  if (packed) return launch_fwd<D, kMaskGeneral, kFeatPacked>(mq, mk, mv, mo, o, lse, p, stream);
  if (p.mask.softcap)
    return launch_fwd<D, kMaskGeneral, kFeatSoftcap>(mq, mk, mv, mo, o, lse, p, stream);
  return launch_fwd<D, kMaskGeneral, 0>(mq, mk, mv, mo, o, lse, p, stream);
}

template <int D>
attn_status dispatch_bwd(const BwdArgs& a, const Problem& p, cudaStream_t stream) {
  using namespace attn;
  if (p.mask.mode == kMaskNone) return launch_bwd<D, kMaskNone, 0>(a, p, stream);
  if (p.mask.mode == kMaskCausal) return launch_bwd<D, kMaskCausal, 0>(a, p, stream);
  const bool packed = p.geom.cu_q != nullptr;
  if (packed && p.mask.softcap)
    return launch_bwd<D, kMaskGeneral, kFeatPacked | kFeatSoftcap>(a, p, stream);
  if (packed) return launch_bwd<D, kMaskGeneral, kFeatPacked>(a, p, stream);
  if (p.mask.softcap) return launch_bwd<D, kMaskGeneral, kFeatSoftcap>(a, p, stream);
  return launch_bwd<D, kMaskGeneral, 0>(a, p, stream);
}

attn_status check_args(const void* const* ptrs, const char* const* names, const bool* used,
                       int n) {
  for (int i = 0; i < n; ++i) {
    if (!used[i]) continue;
    if (ptrs[i] == nullptr) return fail(ATTN_ERR_ARG, "%s is null", names[i]);
    if (!aligned16(ptrs[i])) return fail(ATTN_ERR_ARG, "%s is not 16-byte aligned", names[i]);
  }
  return ATTN_OK;
}

attn_status check_used_ptrs(const void* const* ptrs, const char* const* names, const bool* used,
                            int n) {
  const void* p[16];
  const char* nm[16];
  int m = 0;
  for (int i = 0; i < n && m < 16; ++i)
    if (used[i]) {
      p[m] = ptrs[i];
      nm[m++] = names[i];
    }
  return check_ptrs(p, nm, m);
}

attn_status check_mask_args(int causal, float softcap) {
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  if (!(softcap >= 0.f) || !std::isfinite(softcap))
    return fail(ATTN_ERR_ARG, "softcap must be finite and >= 0 (got %g)", (double)softcap);
  return ATTN_OK;
}

attn::Softcap softcap_consts(float scale, float softcap) {
  if (softcap <= 0.f) return attn::Softcap{0.f, 0.f};
  return attn::Softcap{2.0f * scale * attn::kLog2e / softcap, softcap * attn::kLog2e};
}

// How Q-side and K-side tensors are laid out: TMA map shapes and sizes.
struct Layout {
  long long q_rows, q_z, q_rs, q_zs;   // rows, z extent, row stride, z stride (elements)
  long long k_rows, k_z, k_rs, k_zs;
  long long q_elems, k_elems, lse_elems;
};

// Fixed length: [B, H, N, d], lse [B, Hq, Nq].
void fixed_problem(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int wl,
                   int wr, float softcap, Problem* p, Layout* L) {
  p->B = B; p->Hq = Hq; p->Hkv = Hkv; p->d = d; p->scale = scale;
  p->geom = attn::SeqGeom{nullptr, nullptr, Nq, Nk, 0, 0, static_cast<long long>(Nq) * d, d,
                          static_cast<long long>(Nk) * d, d, Nq};
  p->mask = mask_spec(Nq, Nk, causal, wl, wr, false, softcap);
  p->cap = softcap_consts(scale, softcap);
  *L = Layout{Nq, static_cast<long long>(B) * Hq, d, static_cast<long long>(Nq) * d,
              Nk, static_cast<long long>(B) * Hkv, d, static_cast<long long>(Nk) * d,
              static_cast<long long>(B) * Hq * Nq * d, static_cast<long long>(B) * Hkv * Nk * d,
              static_cast<long long>(B) * Hq * Nq};
}

// Packed: [total, H, d], lse [Hq, total_q], sequences at cu_q / cu_k.
void packed_problem(const int* cu_q, const int* cu_k, int B, int Hq, int Hkv, int total_q,
                    int total_k, int max_q, int max_k, int d, float scale, int causal, int wl,
                    int wr, float softcap, Problem* p, Layout* L) {
  p->B = B; p->Hq = Hq; p->Hkv = Hkv; p->d = d; p->scale = scale;
  p->geom = attn::SeqGeom{cu_q, cu_k, max_q, max_k, total_q, total_k, d,
                          static_cast<long long>(Hq) * d, d, static_cast<long long>(Hkv) * d,
                          total_q};
  p->mask = mask_spec(max_q, max_k, causal, wl, wr, true, softcap);
  p->cap = softcap_consts(scale, softcap);
  *L = Layout{total_q, Hq, static_cast<long long>(Hq) * d, d,
              total_k, Hkv, static_cast<long long>(Hkv) * d, d,
              static_cast<long long>(total_q) * Hq * d, static_cast<long long>(total_k) * Hkv * d,
              static_cast<long long>(Hq) * total_q};
}

// Offsets arrays: null and alignment (host only), then, with a device
// present, that they are device memory.
attn_status check_offsets_args(const int* cu_q, const int* cu_k) {
  const void* ptrs[2] = {cu_q, cu_k};
  const char* names[2] = {"cu_seqlens_q", "cu_seqlens_k"};
  for (int i = 0; i < 2; ++i) {
    if (ptrs[i] == nullptr) return fail(ATTN_ERR_ARG, "%s is null", names[i]);
    if ((reinterpret_cast<uintptr_t>(ptrs[i]) & 3u) != 0)
      return fail(ATTN_ERR_ARG, "%s is not 4-byte aligned", names[i]);
  }
  return ATTN_OK;
}

attn_status check_offsets(const int* cu_q, const int* cu_k) {
  attn_status st = check_device_ptr(cu_q, "cu_seqlens_q");
  if (st != ATTN_OK) return st;
  return check_device_ptr(cu_k, "cu_seqlens_k");
}

// Packed-batch argument checks (host side; offsets are checked on the GPU).
attn_status check_packed(int B, int Hq, int Hkv, int total_q, int total_k, int max_q, int max_k,
                         int d, float scale, bool* no_rows, bool* no_keys) {
  bool e1 = false, e2 = false;
  attn_status st = check_shape(B, Hq, Hkv, max_q, d, scale, &e1);
  if (st != ATTN_OK) return st;
  if ((st = check_shape(B, Hq, Hkv, max_k, d, scale, &e2)) != ATTN_OK) return st;
  if (total_q < 0 || total_k < 0)
    return fail(ATTN_ERR_ARG, "total_q and total_k must be >= 0 (got %d, %d)", total_q, total_k);
  if ((total_q > 0 && max_q == 0) || (total_k > 0 && max_k == 0))
    return fail(ATTN_ERR_ARG, "max_seqlen must be >= 1 when the packed tensor has rows");
  if (static_cast<long long>(total_q) * Hq > 0x7FFFFFFFLL ||
      static_cast<long long>(total_k) * Hkv > 0x7FFFFFFFLL)
    return fail(ATTN_ERR_ARG, "packed tensors too large (total * H must be < 2^31)");
  *no_rows = B == 0 || total_q == 0;
  *no_keys = B == 0 || total_k == 0;
  return ATTN_OK;
}

attn_status fwd_run(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_q, const int* cu_k, const Problem& p, const Layout& L,
                    bool no_rows, bool no_keys, cudaStream_t stream) {
  if (no_rows) return ATTN_OK;                 // no query rows: nothing to write
  const void* ptrs[5] = {q, k, v, o, lse};
  const char* names[5] = {"q", "k", "v", "o", "lse"};
  const bool used[5] = {!no_keys, !no_keys, !no_keys, true, true};
  const bool packed = p.geom.cu_q != nullptr || cu_q != nullptr || cu_k != nullptr;
  attn_status st = check_args(ptrs, names, used, 5);
  if (st != ATTN_OK) return st;
  if (packed && (st = check_offsets_args(cu_q, cu_k)) != ATTN_OK) return st;
  if ((st = ensure_init()) != ATTN_OK) return st;
  if ((st = check_used_ptrs(ptrs, names, used, 5)) != ATTN_OK) return st;
  if (packed && (st = check_offsets(cu_q, cu_k)) != ATTN_OK) return st;
  if (no_keys) {
    // No keys at all: every row sees no key, so O = 0 and lse = -inf.
    cudaError_t e = cudaMemsetAsync(o, 0, static_cast<size_t>(L.q_elems) * 2, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(o)");
    fill_neg_inf_kernel<<<static_cast<unsigned>(std::min<long long>((L.lse_elems + 255) / 256, 4096)),
                          256, 0, stream>>>(lse, L.lse_elems);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "lse fill launch");
    return ATTN_OK;
  }
  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, q, p.d, L.q_rows, L.q_z, L.q_rs, L.q_zs)) != ATTN_OK) return st;
  if ((st = make_map(&mo, o, p.d, L.q_rows, L.q_z, L.q_rs, L.q_zs)) != ATTN_OK) return st;
  if ((st = make_map(&mk, k, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if (p.d == 64) return dispatch_fwd<64>(mq, mk, mv, mo, o, lse, p, stream);
  return dispatch_fwd<128>(mq, mk, mv, mo, o, lse, p, stream);
}

// Backward shared by every backward entry point. With use_static the scratch
// rows live in g_bwd_scratch instead of `workspace`.
attn_status bwd_run(const void* q, const void* k, const void* v, const void* o,
                    const float* lse, const void* dO, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes, bool use_static, const int* cu_q,
                    const int* cu_k, const Problem& p, const Layout& L, bool no_rows,
                    bool no_keys, cudaStream_t stream) {
  if (p.B == 0 || (no_rows && no_keys)) return ATTN_OK;
  const void* ptrs[10] = {q, k, v, o, lse, dO, dq, dk, dv, workspace};
  const char* names[10] = {"q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "workspace"};
  const bool work = !no_rows && !no_keys;
  const bool used[10] = {work, work, work, work, work, work, !no_rows, !no_keys, !no_keys,
                         work && !use_static};
  const bool packed = p.geom.cu_q != nullptr || cu_q != nullptr || cu_k != nullptr;
  attn_status st = check_args(ptrs, names, used, 10);
  if (st != ATTN_OK) return st;
  if (packed && (st = check_offsets_args(cu_q, cu_k)) != ATTN_OK) return st;
  const size_t need = attn_bwd_workspace_size(p.B, p.Hq, p.geom.Nq, p.d);
  if (work && use_static && need > kStaticScratchBytes)
    return fail(ATTN_ERR_ARG,
                "attn_bwd_noalloc: this shape needs %zu bytes of scratch, but the static area "
                "holds %zu (B*Hq*ceil128(N) must be <= %zu); use attn_bwd with a workspace",
                need, kStaticScratchBytes,
                (kStaticScratchBytes - attn::kBwdCounterBytes) / (2 * sizeof(float)));
  if (work && !use_static && workspace_bytes < need)
    return fail(ATTN_ERR_ARG, "workspace is %zu bytes, needs %zu", workspace_bytes, need);
  if ((st = ensure_init()) != ATTN_OK) return st;
  if ((st = check_used_ptrs(ptrs, names, used, 10)) != ATTN_OK) return st;
  if (packed && (st = check_offsets(cu_q, cu_k)) != ATTN_OK) return st;
  if (!work) {
    // No keys: dQ = 0. No queries: dK = dV = 0. (The other side is empty.)
    cudaError_t e = cudaSuccess;
    if (!no_rows) e = cudaMemsetAsync(dq, 0, static_cast<size_t>(L.q_elems) * 2, stream);
    if (e == cudaSuccess && !no_keys)
      e = cudaMemsetAsync(dk, 0, static_cast<size_t>(L.k_elems) * 2, stream);
    if (e == cudaSuccess && !no_keys)
      e = cudaMemsetAsync(dv, 0, static_cast<size_t>(L.k_elems) * 2, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(gradients)");
    return ATTN_OK;
  }
  void* scratch = workspace;
  if (use_static && (st = static_scratch_ptr(&scratch)) != ATTN_OK) return st;
  BwdArgs a;
  if ((st = make_map(&a.mq, q, p.d, L.q_rows, L.q_z, L.q_rs, L.q_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mk, k, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mv, v, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mdo, dO, p.d, L.q_rows, L.q_z, L.q_rs, L.q_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mdk, dk, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mdv, dv, p.d, L.k_rows, L.k_z, L.k_rs, L.k_zs)) != ATTN_OK) return st;
  if ((st = make_map(&a.mdq, dq, p.d, L.q_rows, L.q_z, L.q_rs, L.q_zs)) != ATTN_OK) return st;
  // The preprocess kernel writes every scratch row the other two kernels
  // read, so nothing left from an earlier call is ever used and no clearing
  // is needed (this matters for the static area).
  a.o = o; a.lse = lse; a.dO = dO; a.dq = dq; a.dk = dk; a.dv = dv;
  a.L = static_cast<float*>(scratch);
  a.Dv = a.L + static_cast<size_t>(p.B) * p.Hq * attn::pad128(p.geom.Nq);
  a.sched = reinterpret_cast<int*>(a.Dv + static_cast<size_t>(p.B) * p.Hq * attn::pad128(p.geom.Nq));
  if (p.d == 64) return dispatch_bwd<64>(a, p, stream);
  return dispatch_bwd<128>(a, p, stream);
}

attn_status fwd_fixed(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int wl,
                      int wr, float softcap, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool eq = false, ek = false;
  attn_status st = check_shape(B, Hq, Hkv, Nq, d, scale, &eq);
  if (st != ATTN_OK) return st;
  if ((st = check_shape(B, Hq, Hkv, Nk, d, scale, &ek)) != ATTN_OK) return st;
  if ((st = check_mask_args(causal, softcap)) != ATTN_OK) return st;
  Problem p;
  Layout L;
  fixed_problem(B, Hq, Hkv, Nq, Nk, d, scale, causal, wl, wr, softcap, &p, &L);
  return fwd_run(q, k, v, o, lse, nullptr, nullptr, p, L, eq, ek, stream);
}

attn_status bwd_fixed(const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* dO, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, bool use_static, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int causal, int wl, int wr,
                      float softcap, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool eq = false, ek = false;
  attn_status st = check_shape(B, Hq, Hkv, Nq, d, scale, &eq);
  if (st != ATTN_OK) return st;
  if ((st = check_shape(B, Hq, Hkv, Nk, d, scale, &ek)) != ATTN_OK) return st;
  if ((st = check_mask_args(causal, softcap)) != ATTN_OK) return st;
  Problem p;
  Layout L;
  fixed_problem(B, Hq, Hkv, Nq, Nk, d, scale, causal, wl, wr, softcap, &p, &L);
  return bwd_run(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, use_static, nullptr,
                 nullptr, p, L, eq, ek, stream);
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return 102; }

const char* attn_get_last_error(void) { return g_last_error; }

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal,
                     attn_stream_t stream_) {
  return fwd_fixed(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, -1, -1, 0.f,
                   static_cast<cudaStream_t>(stream_));
}

attn_status attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                            int causal, int window_left, int window_right, float softcap,
                            attn_stream_t stream_) {
  return fwd_fixed(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window_left,
                   window_right, softcap, static_cast<cudaStream_t>(stream_));
}

attn_status attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int Hq,
                            int Hkv, int total_q, int total_k, int max_seqlen_q,
                            int max_seqlen_k, int d, float scale, int causal, int window_left,
                            int window_right, float softcap, attn_stream_t stream_) {
  g_last_error[0] = '\0';
  bool no_rows = false, no_keys = false;
  attn_status st = check_packed(B, Hq, Hkv, total_q, total_k, max_seqlen_q, max_seqlen_k, d,
                                scale, &no_rows, &no_keys);
  if (st != ATTN_OK) return st;
  if ((st = check_mask_args(causal, softcap)) != ATTN_OK) return st;
  Problem p;
  Layout L;
  packed_problem(cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q, total_k, max_seqlen_q,
                 max_seqlen_k, d, scale, causal, window_left, window_right, softcap, &p, &L);
  return fwd_run(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, p, L, no_rows, no_keys,
                 static_cast<cudaStream_t>(stream_));
}

size_t attn_bwd_workspace_size(int B, int Hq, int N, int d) {
  (void)d;
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  // lse * log2(e) and D = rowsum(dO * O), fp32, one row per query padded to
  // a multiple of 128 per head, then the persistent kernels' work counters.
  return 2 * static_cast<size_t>(B) * Hq * attn::pad128(N) * sizeof(float) +
         attn::kBwdCounterBytes;
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dO, void* dq, void* dk, void* dv,
                     void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N,
                     int d, float scale, int causal, attn_stream_t stream_) {
  return bwd_fixed(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, false, B, Hq, Hkv,
                   N, N, d, scale, causal, -1, -1, 0.f, static_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_masked(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                            int Nq, int Nk, int d, float scale, int causal, int window_left,
                            int window_right, float softcap, attn_stream_t stream_) {
  return bwd_fixed(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, false, B, Hq, Hkv,
                   Nq, Nk, d, scale, causal, window_left, window_right, softcap,
                   static_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, void* workspace,
                            size_t workspace_bytes, int B, int Hq, int Hkv, int total_q,
                            int total_k, int max_seqlen_q, int max_seqlen_k, int d, float scale,
                            int causal, int window_left, int window_right, float softcap,
                            attn_stream_t stream_) {
  g_last_error[0] = '\0';
  bool no_rows = false, no_keys = false;
  attn_status st = check_packed(B, Hq, Hkv, total_q, total_k, max_seqlen_q, max_seqlen_k, d,
                                scale, &no_rows, &no_keys);
  if (st != ATTN_OK) return st;
  if ((st = check_mask_args(causal, softcap)) != ATTN_OK) return st;
  Problem p;
  Layout L;
  packed_problem(cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q, total_k, max_seqlen_q,
                 max_seqlen_k, d, scale, causal, window_left, window_right, softcap, &p, &L);
  return bwd_run(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, false, cu_seqlens_q,
                 cu_seqlens_k, p, L, no_rows, no_keys, static_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dO, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             attn_stream_t stream_) {
  return bwd_fixed(q, k, v, o, lse, dO, dq, dk, dv, nullptr, 0, true, B, Hq, Hkv, N, N, d, scale,
                   causal, -1, -1, 0.f, static_cast<cudaStream_t>(stream_));
}


attn_status attn_selftest_wait_timeout(attn_stream_t stream_) {
  g_last_error[0] = '\0';
  attn_status st = ensure_init();
  if (st != ATTN_OK) return st;
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_)>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ATTN_OK;
}

void attn_profile_enable(int on) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  g_prof.on = on != 0;
}

void attn_profile_reset(void) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  for (auto& p : g_prof.pending) {
    g_prof.pool.push_back(p.a);
    g_prof.pool.push_back(p.b);
  }
  g_prof.pending.clear();
  for (int k = 0; k < kProfCount; ++k) {
    g_prof.launches[k] = 0;
    g_prof.total_ms[k] = 0.0;
  }
}

attn_status attn_profile_read(int kernel, const char** name, int* launches, double* total_ms) {
  g_last_error[0] = '\0';
  if (kernel < 0 || kernel >= kProfCount)
    return fail(ATTN_ERR_ARG, "kernel index %d out of range [0, %d)", kernel, (int)kProfCount);
  std::lock_guard<std::mutex> g(g_prof.mu);
  for (auto& p : g_prof.pending) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(p.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.a, p.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event");
    g_prof.launches[p.kernel] += 1;
    g_prof.total_ms[p.kernel] += ms;
    g_prof.pool.push_back(p.a);
    g_prof.pool.push_back(p.b);
  }
  g_prof.pending.clear();
  if (name) *name = kProfNames[kernel];
  if (launches) *launches = g_prof.launches[kernel];
  if (total_ms) *total_ms = g_prof.total_ms[kernel];
  return ATTN_OK;
}

attn_status attn_check_status(attn_stream_t stream_) {
  g_last_error[0] = '\0';
  attn_status st = ensure_init();
  if (st != ATTN_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, attn::g_attn_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(attn::g_attn_device_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
    if ((word & 0xFF) == attn::kDevBadOffsets)
      return fail(ATTN_ERR_ARG,
                  "cu_seqlens offsets out of range (negative, decreasing, past the packed "
                  "tensor, or a sequence longer than max_seqlen); they were clipped");
    return fail(ATTN_ERR_TIMEOUT, "kernel gave up on a pipeline wait (code %d, site %d)",
                word & 0xFF, (word >> 8) & 0xFF);
  }
  return ATTN_OK;
}

}  // extern "C"
