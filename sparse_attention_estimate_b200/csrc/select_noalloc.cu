// select_noalloc.cu - vs_select_noalloc: the vertical-slash selection of
// vs_select for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: a plugin loaded into a
// host application that owns every byte of device memory through its own
// arena, or a service that plans its memory once at start-up and refuses any
// later cudaMalloc. vs_select needs a context whose workspace holds the
// selection thresholds and per-element levels; this entry point keeps that
// scratch instead in one file-scope device array, so the caller passes only
// inputs and outputs and nothing is allocated at call time.
//
// The array lives in the module image: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits (the driver reserves it
// when the library's device code is loaded; with CUDA's lazy module loading
// that happens at the first call here). Its host-side name is only a
// stand-in, so its device address is fetched with cudaGetSymbolAddress, once
// per device and CUDA context, the first time this entry point runs with that
// device current (make that first call before any stream capture begins). The
// address is cached against the context that was current at the lookup: after
// a cudaDeviceReset, or under another context on the same device, the module is
// loaded again at another address, and the next call looks it up again. All
// calls share the array and it keeps the last call's contents; the kernels
// overwrite every byte they read, so nothing needs clearing, but two calls on
// one device whose kernels overlap on the GPU (for example on two streams) race
// on it: serialise them. Each device has its own copy of the array.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.cuh"

namespace vs {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];


// Driver calls through the runtime's driver entry point (no link against libcuda).
template <class Fn>
static Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

// Process-unique id of the current context (0 when none is current). Context ids
// are never reused within a process, unlike context handles.
static unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_ctx = driver_fn<PFN_cuCtxGetCurrent_v4000>("cuCtxGetCurrent");
    get_id = driver_fn<PFN_cuCtxGetId_v12000>("cuCtxGetId");
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device. The lookup (which
// also initialises the device's context and loads the module on first use) runs
// once per device and context: again whenever the current context is not the one
// of the cached lookup, e.g. after cudaDeviceReset.
static vs_status scratch_address(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* addr[kNoAllocMaxDevices] = {};
  static unsigned long long owner[kNoAllocMaxDevices] = {};
  int dev = -1;
  vs_status s = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != VS_OK) return s;
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(VS_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (!addr[dev] || id == 0 || owner[dev] != id) {
    void* p = nullptr;
    s = cuda_check(cudaGetSymbolAddress(&p, g_select_scratch), "cudaGetSymbolAddress(scratch)");
    if (s != VS_OK) return s;
    addr[dev] = static_cast<unsigned char*>(p);
    owner[dev] = current_context_id();  // the context the lookup ran in
  }
  *out = addr[dev];
  return VS_OK;
}

}  // namespace vs

using namespace vs;

extern "C" vs_status vs_select_noalloc(int32_t hq, const float* vert, const float* slash,
                                       int64_t e_ld, int64_t e, const int32_t* kv_budget,
                                       const int32_t* ks_budget, int32_t* v_idx, int32_t cap_v,
                                       int32_t* v_cnt, int32_t* s_off, int32_t cap_s,
                                       int32_t* s_cnt, cudaStream_t stream) {
  if (hq < 1) return set_error(VS_ERR_INVALID_ARG, "hq must be positive");
  if (!vert || !slash || !kv_budget || !ks_budget || !v_idx || !v_cnt || !s_off || !s_cnt)
    return set_error(VS_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (e < 1 || e_ld < e) return set_error(VS_ERR_INVALID_ARG, "need 1 <= e <= e_ld");
  if (cap_v < e || cap_s < e)
    return set_error(VS_ERR_INVALID_ARG, "caps must hold e entries (cap_v, cap_s >= e)");
  // scratch: thresholds, one error word, radix-select state, per-segment histograms,
  // per-element levels of both arrays
  const int64_t e_pad = round_up(e, kTile);
  const size_t thr_bytes = round_up(static_cast<int64_t>(hq) * 2 * kMaxLevels * 2 * 4, 256);
  const size_t err_bytes = 256;
  const size_t state_bytes = round_up(static_cast<int64_t>(sel_state_bytes(hq)), 256);
  const size_t part_bytes = round_up(static_cast<int64_t>(sel_part_bytes(hq, 1)), 256);
  const size_t lvl_bytes = static_cast<size_t>(hq) * 2 * static_cast<size_t>(e_pad);
  const size_t need = thr_bytes + err_bytes + state_bytes + part_bytes + lvl_bytes;
  if (need > kNoAllocScratchBytes)
    return set_error(VS_ERR_UNSUPPORTED,
                     "hq=%d, e=%lld needs %zu bytes of selection scratch; the no-alloc scratch "
                     "holds %zu bytes (use vs_select with a context workspace)",
                     hq, (long long)e, need, kNoAllocScratchBytes);
  unsigned char* base = nullptr;
  vs_status s = scratch_address(&base);
  if (s != VS_OK) return s;
  unsigned char* p = base;
  SelScratch sc{};
  sc.thr = reinterpret_cast<uint32_t*>(p);
  p += thr_bytes;
  sc.err = reinterpret_cast<int*>(p);
  p += err_bytes;
  sc.state = p;
  p += state_bytes;
  sc.part = reinterpret_cast<uint32_t*>(p);
  p += part_bytes;
  sc.lvl = p;
  sc.e_pad = e_pad;
  return launch_select(sc, hq, vert, slash, e_ld, e, kv_budget, ks_budget, 1, nullptr, v_idx, cap_v, v_cnt,
                       s_off, cap_s, s_cnt, true, true, stream);
}
