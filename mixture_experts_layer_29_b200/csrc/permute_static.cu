// permute_static.cu - moe_permute_static_scratch: the permutation step without a
// caller-provided workspace.
//
// Its scratch (the status word, the per-chunk expert bitmasks, their per-expert prefix
// sums and the expert counts) lives in one file-scope __device__ array of a fixed size,
// so the call allocates nothing. Host code may not use the array's name as an address
// (on the host it names a stand-in object, not device memory): the device address is
// looked up with cudaGetSymbolAddress, with the device current, and cached per device
// together with the unique id of the context it was looked up in. A context created
// later on the same device (after cudaDeviceReset, say) has another id, so the address
// is looked up again there. Every call shares the array and it keeps the last call's
// contents.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_permute_scratch[kStaticScratchBytes];

std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};
unsigned long long g_addr_ctx[kMaxDevices] = {};

// The driver's current-context queries, reached through the runtime (no link to libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Unique id of the calling thread's current context (0 if there is none or the driver
// cannot say).
unsigned long long current_context_id() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<CtxGetIdFn>(fn);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!g_ctx_current || !g_ctx_id || g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx ||
      g_ctx_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

inline size_t up1k(size_t v) { return (v + 1023) / 1024 * 1024; }

// Byte offsets inside the static array for this shape: status word, masks, prefixes, counts.
struct StaticLayout {
  size_t masks, crel, ecount, end;
};
StaticLayout static_layout(int T, int n_ffn) {
  const size_t nchunk = (size_t(T) + 31) / 32;
  StaticLayout L;
  L.masks = 1024;
  L.crel = L.masks + up1k(size_t(n_ffn) * nchunk * 4);
  L.ecount = L.crel + up1k(size_t(n_ffn) * nchunk * 4);
  L.end = L.ecount + size_t(n_ffn) * 4;
  return L;
}

// Device address of the array on the current device, looked up the first time a context
// of that device calls here.
int scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  unsigned long long ctx = current_context_id();
  if (!g_addr[dev] || ctx == 0 || g_addr_ctx[dev] != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    ctx = current_context_id();   // the lookup makes the device's context current
    g_addr[dev] = p;
    g_addr_ctx[dev] = ctx;
  }
  *out = g_addr[dev];
  return MOE_OK;
}

inline bool ok_ptr(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_permute_static_scratch(const moe_shape_t* shape, const int32_t* topk_idx,
                                          const float* topk_gate, const float* zgate,
                                          const void* x, int32_t* offsets, int32_t* perm_token,
                                          int32_t* row_of, float* row_gate, void* x_perm,
                                          float* out_acc, void* stream) {
  size_t unused = 0;
  const int rc = moe_scratch_size(shape, &unused);   // the same shape checks as moe_permute
  if (rc != MOE_OK) return rc;
  const void* need[] = {topk_idx, topk_gate, x, offsets, perm_token, row_of, row_gate};
  for (const void* p : need) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(p)) return MOE_ERR_ALIGNMENT;
  }
  if (x_perm && !ok_ptr(x_perm)) return MOE_ERR_ALIGNMENT;   // NULL: indices only, no copy
  if (out_acc) {                          // the zero-expert term needs zgate
    if (!zgate) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(out_acc) || !ok_ptr(zgate)) return MOE_ERR_ALIGNMENT;
  }
  const StaticLayout L = static_layout(shape->T, shape->n_ffn);
  if (L.end > kStaticScratchBytes) return MOE_ERR_WORKSPACE;   // beyond the fixed 4 MiB
  if (shape->T == 0) return MOE_OK;
  DeviceInfo dev;
  const int drc = current_device_info(&dev);
  if (drc != MOE_OK) return drc;
  if (dev.device >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* base = nullptr;
  const int arc = scratch_address(dev.device, &base);
  if (arc != MOE_OK) return arc;
  char* s = static_cast<char*>(base);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word must start at zero; masks, prefixes and counts are fully rewritten
  if (cudaMemsetAsync(s, 0, sizeof(int), st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const cudaError_t e = launch_permute(
      topk_idx, topk_gate, zgate, x, shape->dtype == MOE_BF16, shape->T, shape->H, shape->n_ffn,
      shape->n_ffn + shape->n_zero, shape->K, reinterpret_cast<uint32_t*>(s + L.masks),
      reinterpret_cast<int32_t*>(s + L.crel), reinterpret_cast<int32_t*>(s + L.ecount), offsets,
      perm_token, row_of, row_gate, x_perm, out_acc, reinterpret_cast<int*>(s), st);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
