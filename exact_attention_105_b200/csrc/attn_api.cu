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
#include <mutex>
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
int g_num_sms = 148;
attn_status g_init_status = ATTN_OK;
char g_init_msg[256] = "";
std::once_flag g_init_once;

void init_once() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    g_init_status = ATTN_ERR_CUDA;
    snprintf(g_init_msg, sizeof(g_init_msg), "no CUDA device: %s", cudaGetErrorString(e));
    return;
  }
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess || prop.major != 10 || prop.minor != 0) {
    g_init_status = ATTN_ERR_CUDA;
    snprintf(g_init_msg, sizeof(g_init_msg),
             "this library is built for sm_100a (B200); device %d is sm_%d%d", dev, prop.major,
             prop.minor);
    return;
  }
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) {
    g_init_status = ATTN_ERR_CUDA;
    snprintf(g_init_msg, sizeof(g_init_msg), "cuTensorMapEncodeTiled unavailable");
    return;
  }
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  g_num_sms = prop.multiProcessorCount > 0 ? prop.multiProcessorCount : 148;
}

attn_status ensure_init() {
  std::call_once(g_init_once, init_once);
  if (g_init_status != ATTN_OK) return fail(g_init_status, "%s", g_init_msg);
  return ATTN_OK;
}

// 3-D tensor map over a contiguous [BH, N, d] bf16 tensor with a box of
// 64 x 128 x 1 (one 128-row, 128-byte-wide column block) and 128-byte
// swizzle. Rows past N of a head read as zeros, never as the next head.
attn_status make_map(CUtensorMap* map, const void* base, int d, int N, int BH) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(N)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Null, alignment and memory-kind checks for the tensor arguments. A host
// pointer handed to a kernel would fault the GPU, so it is rejected here.
attn_status check_ptrs(const void* const* ptrs, const char* const* names, int n) {
  for (int i = 0; i < n; ++i) {
    if (ptrs[i] == nullptr) return fail(ATTN_ERR_ARG, "%s is null", names[i]);
    if (!aligned16(ptrs[i])) return fail(ATTN_ERR_ARG, "%s is not 16-byte aligned", names[i]);
  }
  for (int i = 0; i < n; ++i) {
    cudaPointerAttributes pa;
    cudaError_t e = cudaPointerGetAttributes(&pa, ptrs[i]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(ATTN_ERR_ARG, "%s is not a CUDA pointer (%s)", names[i], cudaGetErrorName(e));
    }
    if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)
      return fail(ATTN_ERR_ARG, "%s is not device memory", names[i]);
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
// and causal fast paths.
struct MaskSpec {
  int mode;
  attn::KeyWindow win;
};

MaskSpec mask_spec(int Nq, int Nk, int causal, int window_left, int window_right) {
  using namespace attn;
  const int wl = window_left < 0 ? kUnbounded : std::min(window_left, kUnbounded);
  int wr = window_right < 0 ? kUnbounded : std::min(window_right, kUnbounded);
  if (causal) wr = 0;
  const bool plain = Nq == Nk && wl == kUnbounded && (causal || wr == kUnbounded);
  const int mode = plain ? (causal ? kMaskCausal : kMaskNone) : kMaskGeneral;
  return MaskSpec{mode, KeyWindow{Nk - Nq, wl, wr}};
}

template <int D, int MODE>
attn_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                       attn::KeyWindow win, cudaStream_t stream) {
  using Cfg = attn::FwdCfg<D>;
  auto kern = attn::fwd_kernel<D, MODE>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  static int launch_regs = 0;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmemAlloc);
    cudaFuncAttributes fa;
    if (attr_err == cudaSuccess) attr_err = cudaFuncGetAttributes(&fa, kern);
    if (attr_err == cudaSuccess) launch_regs = fa.numRegs;
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(fwd)");
  // The kernel rebalances registers between warpgroups with setmaxnreg; that
  // split is only valid for the launch register count it was written for.
  if (launch_regs != attn::kFwdRegsLaunch)
    return fail(ATTN_ERR_CUDA, "fwd kernel built with %d registers/thread, expected %d",
                launch_regs, attn::kFwdRegsLaunch);
  const long long blocks = static_cast<long long>(B) * Hq * ((Nq + 255) / 256);
  if (blocks > 0x7FFFFFFFLL) return fail(ATTN_ERR_ARG, "problem too large for one launch");
  dim3 grid(static_cast<unsigned>(blocks));
  const float scale_log2 = scale * 1.4426950408889634f;
  ProfScope ps(kProfFwd, stream);
  kern<<<grid, Cfg::kThreads, Cfg::kSmemAlloc, stream>>>(
      mq, mk, mv, static_cast<__nv_bfloat16*>(o), lse, Hq, Hq / Hkv, Nq, Nk, scale_log2, win);
  ps.end();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fwd kernel launch");
  return ATTN_OK;
}

// One-time per-kernel setup: opt in to the dynamic shared memory size.
template <typename Kern>
cudaError_t set_smem_once(Kern kern, int bytes, std::once_flag& once, cudaError_t& err) {
  std::call_once(once, [&] {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return err;
}

struct BwdArgs {
  CUtensorMap mq, mk, mv, mdo;
  const void* o;
  const float* lse;
  const void* dO;
  void *dq, *dk, *dv;
  float *L, *Dv;
  int B, Hq, Hkv, Nq, Nk;
  float scale;
  attn::KeyWindow win;
};

template <int D, int MODE>
attn_status launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  using namespace attn;
  const int Npad = pad128(a.Nq);
  const int group = a.Hq / a.Hkv;
  const float scale_log2 = a.scale * kLog2e;

  const long long rows = static_cast<long long>(a.B) * a.Hq * Npad;
  const long long g1 = static_cast<long long>(pad128(a.Nk) / 128) * a.B * a.Hkv;
  const long long g2 = static_cast<long long>(Npad / 128) * a.B * a.Hq;
  if (rows / 32 > 0x7FFFFFFFLL) return fail(ATTN_ERR_ARG, "problem too large for one launch");
  ProfScope p0(kProfBwdPre, stream);
  bwd_pre_kernel<D><<<static_cast<unsigned>(rows / 32), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dO), a.lse,
      a.L, a.Dv, a.Nq, Npad);
  p0.end();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd preprocess launch");

  static std::once_flag o1, o2;
  static cudaError_t e1 = cudaSuccess, e2 = cudaSuccess;
  auto k1 = bwd_dkdv_kernel<D, MODE>;
  auto k2 = bwd_dq_kernel<D, MODE>;
  if ((e = set_smem_once(k1, DkdvCfg<D>::kSmemAlloc, o1, e1)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(dkdv)");
  if ((e = set_smem_once(k2, DqCfg<D>::kSmemAlloc, o2, e2)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(dq)");

  ProfScope p1(kProfBwdDkdv, stream);
  k1<<<dim3(static_cast<unsigned>(g1)), DkdvCfg<D>::kThreads, DkdvCfg<D>::kSmemAlloc, stream>>>(
      a.mq, a.mk, a.mv, a.mdo, a.L, a.Dv, static_cast<__nv_bfloat16*>(a.dk),
      static_cast<__nv_bfloat16*>(a.dv), a.Hq, group, a.Nq, a.Nk, Npad, scale_log2, a.scale,
      a.win);
  p1.end();
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd dK/dV launch");
  ProfScope p2(kProfBwdDq, stream);
  k2<<<dim3(static_cast<unsigned>(g2)), DqCfg<D>::kThreads, DqCfg<D>::kSmemAlloc, stream>>>(
      a.mq, a.mk, a.mv, a.mdo, a.L, a.Dv, static_cast<__nv_bfloat16*>(a.dq), a.Hq, group, a.Nq,
      a.Nk, Npad, scale_log2, a.scale, a.win);
  p2.end();
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd dQ launch");
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
// 8 MiB until the process exits. Host code must not hand the symbol itself to
// a kernel (on the host it names a stand-in, not device memory). Its device
// address is looked up once per device with cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) float g_bwd_scratch[kStaticScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
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
                         void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                         const MaskSpec& m, cudaStream_t stream) {
  using namespace attn;
  if (m.mode == kMaskNone)
    return launch_fwd<D, kMaskNone>(mq, mk, mv, o, lse, B, Hq, Hkv, Nq, Nk, scale, m.win, stream);
  if (m.mode == kMaskCausal)
    return launch_fwd<D, kMaskCausal>(mq, mk, mv, o, lse, B, Hq, Hkv, Nq, Nk, scale, m.win,
                                      stream);
  return launch_fwd<D, kMaskGeneral>(mq, mk, mv, o, lse, B, Hq, Hkv, Nq, Nk, scale, m.win, stream);
}

template <int D>
attn_status dispatch_bwd(const BwdArgs& a, int mode, cudaStream_t stream) {
  using namespace attn;
  if (mode == kMaskNone) return launch_bwd<D, kMaskNone>(a, stream);
  if (mode == kMaskCausal) return launch_bwd<D, kMaskCausal>(a, stream);
  return launch_bwd<D, kMaskGeneral>(a, stream);
}

attn_status check_common(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         bool* no_rows, bool* no_keys) {
  bool eq = false, ek = false;
  attn_status st = check_shape(B, Hq, Hkv, Nq, d, scale, &eq);
  if (st != ATTN_OK) return st;
  if ((st = check_shape(B, Hq, Hkv, Nk, d, scale, &ek)) != ATTN_OK) return st;
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  *no_rows = eq;
  *no_keys = ek;
  return ATTN_OK;
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

attn_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     int window_left, int window_right, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool no_rows = false, no_keys = false;
  attn_status st = check_common(B, Hq, Hkv, Nq, Nk, d, scale, causal, &no_rows, &no_keys);
  if (st != ATTN_OK) return st;
  if (no_rows) return ATTN_OK;                 // B == 0 or Nq == 0: nothing to write
  const void* ptrs[5] = {q, k, v, o, lse};
  const char* names[5] = {"q", "k", "v", "o", "lse"};
  const bool used[5] = {!no_keys, !no_keys, !no_keys, true, true};
  if ((st = check_args(ptrs, names, used, 5)) != ATTN_OK) return st;
  if ((st = ensure_init()) != ATTN_OK) return st;
  if ((st = check_used_ptrs(ptrs, names, used, 5)) != ATTN_OK) return st;
  if (no_keys) {
    // Nk == 0: every row sees no key, so O = 0 and lse = -inf.
    const long long rows = static_cast<long long>(B) * Hq * Nq;
    cudaError_t e = cudaMemsetAsync(o, 0, static_cast<size_t>(rows) * d * 2, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(o)");
    fill_neg_inf_kernel<<<static_cast<unsigned>(std::min<long long>((rows + 255) / 256, 4096)),
                          256, 0, stream>>>(lse, rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "lse fill launch");
    return ATTN_OK;
  }
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, d, Nq, B * Hq)) != ATTN_OK) return st;
  if ((st = make_map(&mk, k, d, Nk, B * Hkv)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v, d, Nk, B * Hkv)) != ATTN_OK) return st;
  const MaskSpec m = mask_spec(Nq, Nk, causal, window_left, window_right);
  if (d == 64) return dispatch_fwd<64>(mq, mk, mv, o, lse, B, Hq, Hkv, Nq, Nk, scale, m, stream);
  return dispatch_fwd<128>(mq, mk, mv, o, lse, B, Hq, Hkv, Nq, Nk, scale, m, stream);
}

// Backward shared by attn_bwd, attn_bwd_masked and attn_bwd_noalloc. With
// use_static the scratch rows live in g_bwd_scratch instead of `workspace`.
attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dO, void* dq, void* dk, void* dv,
                     void* workspace, size_t workspace_bytes, bool use_static, int B, int Hq,
                     int Hkv, int Nq, int Nk, int d, float scale, int causal, int window_left,
                     int window_right, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool no_rows = false, no_keys = false;
  attn_status st = check_common(B, Hq, Hkv, Nq, Nk, d, scale, causal, &no_rows, &no_keys);
  if (st != ATTN_OK) return st;
  if (B == 0 || (no_rows && no_keys)) return ATTN_OK;
  const void* ptrs[10] = {q, k, v, o, lse, dO, dq, dk, dv, workspace};
  const char* names[10] = {"q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "workspace"};
  const bool work = !no_rows && !no_keys;
  const bool used[10] = {work, work, work, work, work, work, !no_rows, !no_keys, !no_keys,
                         work && !use_static};
  if ((st = check_args(ptrs, names, used, 10)) != ATTN_OK) return st;
  const size_t need = attn_bwd_workspace_size(B, Hq, Nq, d);
  if (work && use_static && need > kStaticScratchBytes)
    return fail(ATTN_ERR_ARG,
                "attn_bwd_noalloc: this shape needs %zu bytes of scratch, but the static area "
                "holds %zu (B*Hq*ceil128(N) must be <= %zu); use attn_bwd with a workspace",
                need, kStaticScratchBytes, kStaticScratchBytes / (2 * sizeof(float)));
  if (work && !use_static && workspace_bytes < need)
    return fail(ATTN_ERR_ARG, "workspace is %zu bytes, needs %zu", workspace_bytes, need);
  if ((st = ensure_init()) != ATTN_OK) return st;
  if ((st = check_used_ptrs(ptrs, names, used, 10)) != ATTN_OK) return st;
  if (!work) {
    // No keys: dQ = 0. No queries: dK = dV = 0. (The other side is empty.)
    const size_t kv_bytes = static_cast<size_t>(B) * Hkv * Nk * d * 2;
    const size_t q_bytes = static_cast<size_t>(B) * Hq * Nq * d * 2;
    cudaError_t e = cudaSuccess;
    if (!no_rows) e = cudaMemsetAsync(dq, 0, q_bytes, stream);
    if (e == cudaSuccess && !no_keys) e = cudaMemsetAsync(dk, 0, kv_bytes, stream);
    if (e == cudaSuccess && !no_keys) e = cudaMemsetAsync(dv, 0, kv_bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(gradients)");
    return ATTN_OK;
  }
  void* scratch = workspace;
  if (use_static && (st = static_scratch_ptr(&scratch)) != ATTN_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_map(&mq, q, d, Nq, B * Hq)) != ATTN_OK) return st;
  if ((st = make_map(&mk, k, d, Nk, B * Hkv)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v, d, Nk, B * Hkv)) != ATTN_OK) return st;
  if ((st = make_map(&mdo, dO, d, Nq, B * Hq)) != ATTN_OK) return st;
  // The preprocess kernel writes every scratch row the other two kernels
  // read, so nothing left from an earlier call is ever used and no clearing
  // is needed (this matters for the static area).
  float* L = static_cast<float*>(scratch);
  float* Dv = L + static_cast<size_t>(B) * Hq * attn::pad128(Nq);
  const MaskSpec m = mask_spec(Nq, Nk, causal, window_left, window_right);
  BwdArgs a{mq, mk, mv, mdo, o, lse, dO, dq, dk, dv, L, Dv, B, Hq, Hkv, Nq, Nk, scale, m.win};
  if (d == 64) return dispatch_bwd<64>(a, m.mode, stream);
  return dispatch_bwd<128>(a, m.mode, stream);
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return 101; }

const char* attn_get_last_error(void) { return g_last_error; }

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal,
                     attn_stream_t stream_) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, -1, -1,
                  static_cast<cudaStream_t>(stream_));
}

attn_status attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                            int causal, int window_left, int window_right,
                            attn_stream_t stream_) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window_left,
                  window_right, static_cast<cudaStream_t>(stream_));
}

size_t attn_bwd_workspace_size(int B, int Hq, int N, int d) {
  (void)d;
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  // lse * log2(e) and D = rowsum(dO * O), fp32, one row per query padded to
  // a multiple of 128 per head.
  return 2 * static_cast<size_t>(B) * Hq * attn::pad128(N) * sizeof(float);
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dO, void* dq, void* dk, void* dv,
                     void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N,
                     int d, float scale, int causal, attn_stream_t stream_) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, false, B, Hq, Hkv,
                  N, N, d, scale, causal, -1, -1, static_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_masked(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                            int Nq, int Nk, int d, float scale, int causal, int window_left,
                            int window_right, attn_stream_t stream_) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, false, B, Hq, Hkv,
                  Nq, Nk, d, scale, causal, window_left, window_right,
                  static_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dO, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             attn_stream_t stream_) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, nullptr, 0, true, B, Hq, Hkv, N, N, d, scale,
                  causal, -1, -1, static_cast<cudaStream_t>(stream_));
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
    return fail(ATTN_ERR_TIMEOUT, "kernel gave up on a pipeline wait (code %d, site %d)",
                word & 0xFF, (word >> 8) & 0xFF);
  }
  return ATTN_OK;
}

}  // extern "C"
