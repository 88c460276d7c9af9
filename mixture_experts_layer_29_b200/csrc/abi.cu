// abi.cu - the extern "C" entry points of include/moe.h: host-side argument checks, the
// workspace layout and the launch order of the layer's kernels. No call here allocates
// device memory or waits for the device, except moe_read_device_status and the host
// pipeline's create (streams and events) and destroy (waits for its copies).
#include <atomic>
#include <initializer_list>
#include <mutex>
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Process-wide tuning switches (moe_set_tuning), each at its default until changed.
namespace {
constexpr int kTuneCount = MOE_TUNE_BWD_WGRAD_BK + 1;
std::atomic<int64_t> g_tune[kTuneCount] = {{1}, {-1}, {1}, {0}, {12}, {1}, {4}, {0}, {0}, {0}, {0}, {1},
                                           {1}, {1}, {0}, {0}, {16}, {0}, {64}};

bool tune_value_ok(int knob, int64_t v) {
  switch (knob) {
    case MOE_TUNE_BWD_PAIR: return v >= 0 && v <= 2;
    case MOE_TUNE_PDL:
    case MOE_TUNE_PAIR_HALF:
    case MOE_TUNE_PAIR_INTERLEAVE:
    case MOE_TUNE_PAIR_A_TRIM:
    case MOE_TUNE_PAIR_SWAP_AB:
    case MOE_TUNE_PAIR_STREAM_HINT:
    case MOE_TUNE_PAIR_TAILS:
    case MOE_TUNE_TEST_STALL: return v == 0 || v == 1;
    case MOE_TUNE_GEMM_PAIR: return v >= -1 && v <= 1;
    case MOE_TUNE_ROUTER_N: return v == 0 || v == 192 || v == 256;
    case MOE_TUNE_ROUTER_MIN_SPLIT: return v >= 1 && v <= 1024;
    case MOE_TUNE_BWD_DY_ROWS: return v == 1 || v == 4;
    case MOE_TUNE_GATE_UP_BAND:
    case MOE_TUNE_DOWN_BAND:
    case MOE_TUNE_PAIR_PREFETCH: return v >= 0 && v <= 64;
    case MOE_TUNE_BWD_WGRAD_GROUP: return v >= 0 && v <= 64;
    case MOE_TUNE_BWD_WGRAD_MIX: return v >= 0 && v <= 65536;
    case MOE_TUNE_BWD_WGRAD_BK: return v == 64 || v == 128;
    default: return false;
  }
}
}  // namespace

int64_t tuning(int knob) { return g_tune[knob].load(std::memory_order_relaxed); }

bool take_test_stall() { return g_tune[MOE_TUNE_TEST_STALL].exchange(0) != 0; }

bool pdl_enabled() { return tuning(MOE_TUNE_PDL) != 0; }

int current_device_info(DeviceInfo* info) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].device != dev) {
    DeviceInfo d;
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    cache[dev] = d;
  }
  *info = cache[dev];
  // the kernels are built for sm_100a only
  if (info->cc_major != 10 || info->cc_minor != 0) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

namespace {

constexpr size_t kAlign = 1024;
constexpr int kRowPad = 128;    // extra rows of x_perm / h / y_perm read by the GEMM tiles

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  // scratch (all step calls)
  size_t status, masks, crel, ecount, lbpart, lpart, scratch_end;
  // intermediates (moe_forward)
  size_t logits, zgate, offsets, perm, rowof, rowgate, xperm, h, yperm, outacc, total;
};

int check_shape(const moe_shape_t* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->I <= 0 || s->n_ffn <= 0 || s->n_zero < 0 || s->K <= 0)
    return MOE_ERR_INVALID_ARG;
  if (s->dtype != MOE_BF16 && s->dtype != MOE_FP32) return MOE_ERR_INVALID_ARG;
  if (s->combine != MOE_COMBINE_FUSED && s->combine != MOE_COMBINE_DETERMINISTIC)
    return MOE_ERR_INVALID_ARG;
  const long E = (long)s->n_ffn + s->n_zero;
  if (s->K > E) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || s->K > 32) return MOE_ERR_UNSUPPORTED;
  if (s->T >= (1 << 24) || (long)s->T * s->K >= (1L << 31)) return MOE_ERR_UNSUPPORTED;
  if (s->H % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (s->dtype == MOE_BF16 && (s->H % 128 != 0 || s->I % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (!(s->ffn_out_scale == s->ffn_out_scale)) return MOE_ERR_INVALID_ARG;   // NaN
  return MOE_OK;
}

Layout layout_of(const moe_shape_t& s) {
  Layout L{};
  const size_t T = s.T, H = s.H, I = s.I, N = s.n_ffn, K = s.K, E = N + s.n_zero;
  const size_t nchunk = (T + 31) / 32;
  const size_t esz = s.dtype == MOE_BF16 ? 2 : 4;
  const size_t rows = T * K + kRowPad;
  size_t o = 0;
  L.status = o;  o = align_up(o + 256);
  L.masks = o;   o = align_up(o + N * nchunk * 4);
  L.crel = o;    o = align_up(o + N * nchunk * 4);
  L.ecount = o;  o = align_up(o + N * 4);
  L.lbpart = o;  o = align_up(o + lb_partial_bytes(s.T, (int)E));
  L.lpart = o;   // router scratch: split weight + partials (bf16) or SIMT partials (fp32)
  o = align_up(o + (s.dtype == MOE_BF16 ? router_tc_scratch_bytes(s.T, (int)E, s.H)
                                        : router_partial_bytes(s.T, (int)E, s.H, 0)));
  L.scratch_end = o;
  L.logits = o;  o = align_up(o + T * E * 4);
  L.zgate = o;   o = align_up(o + T * 4);
  L.offsets = o; o = align_up(o + (N + 1) * 4);
  L.perm = o;    o = align_up(o + T * K * 4);
  L.rowof = o;   o = align_up(o + T * K * 4);
  L.rowgate = o; o = align_up(o + T * K * 4);
  L.xperm = o;   o = align_up(o + rows * H * esz);
  L.h = o;       o = align_up(o + rows * I * esz);
  L.yperm = o;
  if (s.combine == MOE_COMBINE_DETERMINISTIC) o = align_up(o + rows * H * esz);
  L.outacc = o;
  if (s.combine == MOE_COMBINE_FUSED) o = align_up(o + T * H * 4);
  L.total = o;
  return L;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// all given pointers non-null and 16-byte aligned
int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
  }
  return MOE_OK;
}
// optional pointers: may be null, else aligned
int check_opt(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)            \
  do {                           \
    const int _rc = (expr);      \
    if (_rc != MOE_OK) return _rc; \
  } while (0)

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int route_impl(const moe_shape_t* s, const void* x, const float* w_router, const void* w_packed,
               const float* logits_in, const float* bias, float* logits_out, int32_t* topk_idx,
               float* topk_gate, int32_t* counts, int32_t* nffn_hist, float* zgate, void* ws,
               size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(s));
  MOE_TRY(check_ptrs({bias, topk_idx, topk_gate, counts, nffn_hist, zgate, ws}));
  if (!logits_in) MOE_TRY(check_ptrs({x, w_packed ? w_packed : w_router, logits_out}));
  if (w_packed && s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_opt({logits_in, logits_out, x, w_router}));
  const Layout L = layout_of(*s);
  if (ws_bytes < L.scratch_end) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  const int E = s->n_ffn + s->n_zero;
  const cudaStream_t st = as_stream(stream);
  const float* src = logits_in;      // logits, or S split-K slices of them
  int S = 1;
  // the router kernel clears the counts and the histogram the top-K kernel adds to
  ZeroSpec zero;
  zero.a = counts;
  zero.na = E;
  zero.b = nffn_hist;
  zero.nb = s->K + 1;
  if (!logits_in) {
    if (s->dtype == MOE_BF16) {
      MOE_TRY(launch_router_logits_tc(x, w_router, w_packed, s->T, E, s->H, logits_out,
                                      at<char>(ws, L.lpart), dev.sm_count, zero, st, &src, &S));
    } else {
      S = router_splitk(s->T, E, s->H, dev.sm_count);
      float* part = at<float>(ws, L.lpart);
      MOE_TRY(cuda_rc(launch_router_logits(x, 0, w_router, s->T, E, s->H, logits_out, part, S,
                                           zero, st)));
      src = S > 1 ? part : logits_out;
    }
  } else {
    MOE_TRY(cuda_rc(launch_zero_counts(counts, E, nffn_hist, s->K, st)));
  }
  if (!route_topk_sums_slices(s->T, S, dev.sm_count)) {
    // many slices and many tokens: one wide reduction kernel first
    MOE_TRY(cuda_rc(launch_splitk_sum(src, S, (size_t)s->T * E, logits_out, st)));
    src = logits_out;
    S = 1;
  }
  return cuda_rc(launch_route_topk(src, S, logits_out, bias, s->T, E, s->n_ffn, s->K, topk_idx,
                                   topk_gate, counts, nffn_hist, zgate, dev.sm_count, st));
}

int permute_impl(const moe_shape_t* s, const int32_t* topk_idx, const float* topk_gate,
                 const float* zgate, const void* x, int32_t* offsets, int32_t* perm_token,
                 int32_t* row_of, float* row_gate, void* x_perm, float* out_acc, void* ws,
                 size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(s));
  MOE_TRY(check_ptrs({topk_idx, topk_gate, x, offsets, perm_token, row_of, row_gate, ws}));
  MOE_TRY(check_opt({x_perm}));
  if (out_acc) MOE_TRY(check_ptrs({zgate, out_acc}));
  const Layout L = layout_of(*s);
  if (ws_bytes < L.scratch_end) return MOE_ERR_WORKSPACE;
  if (s->T == 0) {
    return MOE_OK;
  }
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  return cuda_rc(launch_permute(topk_idx, topk_gate, zgate, x, s->dtype == MOE_BF16, s->T, s->H,
                                s->n_ffn, s->n_ffn + s->n_zero, s->K, at<uint32_t>(ws, L.masks),
                                at<int32_t>(ws, L.crel), at<int32_t>(ws, L.ecount), offsets,
                                perm_token, row_of, row_gate, x_perm, out_acc,
                                at<int>(ws, L.status), as_stream(stream)));
}

int grouped_ffn_impl(const moe_shape_t* s, const void* x, const void* x_perm,
                     const int32_t* offsets, const void* w_gate_up, const void* w_down,
                     const int32_t* perm_token, const float* row_gate, void* h, void* y_perm,
                     float* out_acc, void* gu_out, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(s));
  MOE_TRY(check_ptrs({offsets, w_gate_up, w_down, h, ws}));
  MOE_TRY(check_opt({gu_out}));
  if (gu_out && s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (x_perm) MOE_TRY(check_ptrs({x_perm}));
  else if (s->dtype == MOE_BF16) MOE_TRY(check_ptrs({x, perm_token}));   // gathered rows
  else return MOE_ERR_INVALID_ARG;                                      // fp32 needs x_perm
  const bool fused = s->combine == MOE_COMBINE_FUSED;
  if (fused) MOE_TRY(check_ptrs({perm_token, row_gate, out_acc}));
  else MOE_TRY(check_ptrs({y_perm}));
  const Layout L = layout_of(*s);
  if (ws_bytes < L.scratch_end) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  const cudaStream_t st = as_stream(stream);
  if (s->dtype == MOE_BF16)
    return launch_grouped_ffn_tc(x, x_perm, offsets, w_gate_up, w_down, perm_token, row_gate, h, y_perm,
                                 out_acc, gu_out, s->T, s->H, s->I, s->n_ffn, s->K, s->ffn_out_scale, fused,
                                 at<int>(ws, L.status), dev.sm_count, st);
  return cuda_rc(launch_grouped_ffn_simt(
      static_cast<const float*>(x_perm), offsets, static_cast<const float*>(w_gate_up),
      static_cast<const float*>(w_down), perm_token, row_gate, static_cast<float*>(h),
      static_cast<float*>(y_perm), out_acc, s->T, s->H, s->I, s->n_ffn, s->K, s->ffn_out_scale,
      fused, st));
}

int combine_impl(const moe_shape_t* s, const void* x, const void* y_perm, const float* out_acc,
                 const float* topk_gate, const int32_t* row_of, const float* zgate, void* out,
                 void* stream) {
  MOE_TRY(check_shape(s));
  MOE_TRY(check_ptrs({out}));
  const bool fused = s->combine == MOE_COMBINE_FUSED;
  if (fused) MOE_TRY(check_ptrs({out_acc}));
  else MOE_TRY(check_ptrs({x, y_perm, topk_gate, row_of, zgate}));
  if (s->T == 0) return MOE_OK;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  const cudaStream_t st = as_stream(stream);
  if (fused)
    return cuda_rc(launch_finalize(out_acc, out, s->dtype == MOE_BF16, (size_t)s->T * s->H, st));
  return cuda_rc(launch_combine_det(x, y_perm, topk_gate, row_of, zgate, out, s->dtype == MOE_BF16,
                                    s->T, s->H, s->K, s->ffn_out_scale, st));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_scratch_size(const moe_shape_t* shape, size_t* bytes) {
  MOE_TRY(check_shape(shape));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = layout_of(*shape).scratch_end;
  return MOE_OK;
}

int moe_workspace_size(const moe_shape_t* shape, size_t* bytes) {
  MOE_TRY(check_shape(shape));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = layout_of(*shape).total;
  return MOE_OK;
}

// Backward workspace: status word, G|U, dy, dG|dU, dx_perm (fp32), the picks' gate
// gradients and the logit gradient.
struct BwdLayout {
  size_t status, offs, gu, dy, dgu, dxp, dgate, dl3, wr16, total;
};

static BwdLayout bwd_layout_of(const moe_shape_t& s) {
  BwdLayout L{};
  const size_t T = s.T, H = s.H, I = s.I, K = s.K, E = (size_t)s.n_ffn + s.n_zero;
  const size_t rows = T * K + kRowPad;
  size_t o = 0;
  const size_t Tp = (T + 63) / 64 * 64;
  L.status = o; o = align_up(o + 256);
  L.offs = o;   o = align_up(o + 4 * 4);
  L.gu = o;     o = align_up(o + rows * 2 * I * 2);
  L.dy = o;     o = align_up(o + rows * H * 2);
  L.dgu = o;    o = align_up(o + rows * 2 * I * 2);
  L.dxp = o;    o = align_up(o + rows * H * 4);
  L.dgate = o;  o = align_up(o + T * K * 4);
  L.dl3 = o;    o = align_up(o + 3 * Tp * E * 2);
  L.wr16 = o;   o = align_up(o + E * (size_t)s.H * 2);
  L.total = o;
  return L;
}

int moe_backward_workspace_size(const moe_shape_t* shape, size_t* bytes) {
  MOE_TRY(check_shape(shape));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = bwd_layout_of(*shape).total;
  return MOE_OK;
}

int moe_backward(const moe_shape_t* shape, const void* dout, const void* x,
                 const float* w_router, const void* w_gate_up, const void* w_down,
                 const float* logits, const int32_t* topk_idx, const float* topk_gate,
                 const int32_t* offsets, const int32_t* row_of, const void* x_perm,
                 const void* h, const void* y_perm, const void* gu_saved, float* dx,
                 float* d_router, float* d_gate_up, float* d_down, void* ws, size_t ws_bytes,
                 void* stream) {
  MOE_TRY(check_shape(shape));
  if (shape->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if ((shape->n_ffn + shape->n_zero) % 8 != 0) return MOE_ERR_UNSUPPORTED;   // dL rows: 16 B
  MOE_TRY(check_ptrs({dout, x, w_router, w_gate_up, w_down, logits, topk_idx, topk_gate, offsets,
                      row_of, x_perm, h, y_perm, dx, d_router, d_gate_up, d_down, ws}));
  MOE_TRY(check_opt({gu_saved}));
  const BwdLayout L = bwd_layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (shape->T == 0) return MOE_OK;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  const cudaStream_t st = as_stream(stream);
  const int T = shape->T, H = shape->H, I = shape->I, K = shape->K, N = shape->n_ffn;
  const int E = N + shape->n_zero;
  int* status = at<int>(ws, L.status);
  const void* gu = gu_saved ? gu_saved : at<char>(ws, L.gu);
  void* dy = at<char>(ws, L.dy);
  void* dgu = at<char>(ws, L.dgu);
  float* dxp = at<float>(ws, L.dxp);
  float* dgate = at<float>(ws, L.dgate);
  void* dl3 = at<char>(ws, L.dl3);
  void* wr16 = at<char>(ws, L.wr16);
  int32_t* offs = at<int32_t>(ws, L.offs);
  const int Tp = (T + 63) / 64 * 64;
  // G | U of every FFN row again (unless the forward saved them), then dy and the gates'
  // gradients
  if (!gu_saved)
    MOE_TRY(launch_gate_up_raw(x_perm, offsets, w_gate_up, at<char>(ws, L.gu), T, H, I, N, K,
                               status, dev.sm_count, st));
  MOE_TRY(cuda_rc(launch_bwd_dy_dgate(dout, x, y_perm, topk_idx, topk_gate, row_of, T, H, K, N,
                                      shape->ffn_out_scale, dy, dgate, st)));
  // the expert GEMMs: dgu (with the SwiGLU backward), dx_perm, d_down, d_gate_up
  MOE_TRY(launch_bwd_gemms(dy, gu, h, x_perm, offsets, w_gate_up, w_down, dgu, dxp, d_gate_up,
                           d_down, T, H, I, N, K, status, dev.sm_count, st));
  // router: logit gradient (three bf16 parts), d_router = dL^T x, dx = dL W_r; then the
  // rows' gradients and the zero-expert term
  MOE_TRY(cuda_rc(launch_bwd_router(logits, topk_idx, dgate, T, Tp, E, K, dl3, offs, w_router,
                                    wr16, H, st)));
  MOE_TRY(launch_bwd_router_gemms(dl3, Tp, x, wr16, offs, offs + 2, T, E, H, d_router, dx,
                                  status, dev.sm_count, st));
  return cuda_rc(launch_bwd_dx_combine(dxp, dout, topk_idx, topk_gate, row_of, T, H, K, N, dx, st));
}

int moe_read_device_status(void* ws, size_t ws_bytes, void* stream, int32_t* status) {
  if (!ws || !status) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < 256) return MOE_ERR_WORKSPACE;
  const cudaStream_t st = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(ws, 0, sizeof(v), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *status = v;
  return MOE_OK;
}

const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_DEVICE_CHECK: return "device-side consistency check failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_NO_DEVICE: return "no sm_100 CUDA device";
    default: return "unknown status";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_set_tuning(int knob, int64_t value) {
  if (knob < 0 || knob >= kTuneCount || !tune_value_ok(knob, value)) return MOE_ERR_INVALID_ARG;
  g_tune[knob].store(value, std::memory_order_relaxed);
  return MOE_OK;
}

int moe_get_tuning(int knob, int64_t* value) {
  if (knob < 0 || knob >= kTuneCount || !value) return MOE_ERR_INVALID_ARG;
  *value = tuning(knob);
  return MOE_OK;
}

int moe_route(const moe_shape_t* shape, const void* x, const float* w_router,
              const float* logits_in, const float* bias, float* logits_out, int32_t* topk_idx,
              float* topk_gate, int32_t* counts, int32_t* nffn_hist, float* zgate, void* ws,
              size_t ws_bytes, void* stream) {
  return route_impl(shape, x, w_router, nullptr, logits_in, bias, logits_out, topk_idx, topk_gate,
                    counts, nffn_hist, zgate, ws, ws_bytes, stream);
}

int moe_router_pack(const moe_shape_t* shape, const float* w_router, void* w_packed,
                    void* stream) {
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({w_router, w_packed}));
  if (shape->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  return launch_router_pack(w_router, w_packed, shape->n_ffn + shape->n_zero, shape->H,
                            dev.sm_count, as_stream(stream));
}

int moe_route_packed(const moe_shape_t* shape, const void* x, const void* w_packed,
                     const float* bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
                     int32_t* counts, int32_t* nffn_hist, float* zgate, void* ws, size_t ws_bytes,
                     void* stream) {
  if (!w_packed) return MOE_ERR_INVALID_ARG;
  return route_impl(shape, x, nullptr, w_packed, nullptr, bias, logits_out, topk_idx, topk_gate,
                    counts, nffn_hist, zgate, ws, ws_bytes, stream);
}

int moe_permute(const moe_shape_t* shape, const int32_t* topk_idx, const float* topk_gate,
                const float* zgate, const void* x, int32_t* offsets, int32_t* perm_token,
                int32_t* row_of, float* row_gate, void* x_perm, float* out_acc, void* ws,
                size_t ws_bytes, void* stream) {
  return permute_impl(shape, topk_idx, topk_gate, zgate, x, offsets, perm_token, row_of, row_gate,
                      x_perm, out_acc, ws, ws_bytes, stream);
}

int moe_grouped_ffn(const moe_shape_t* shape, const void* x, const void* x_perm,
                    const int32_t* offsets, const void* w_gate_up, const void* w_down,
                    const int32_t* perm_token, const float* row_gate, void* h, void* y_perm,
                    float* out_acc, void* gu_out, void* ws, size_t ws_bytes, void* stream) {
  return grouped_ffn_impl(shape, x, x_perm, offsets, w_gate_up, w_down, perm_token, row_gate, h,
                          y_perm, out_acc, gu_out, ws, ws_bytes, stream);
}

int moe_combine(const moe_shape_t* shape, const void* x, const void* y_perm, const float* out_acc,
                const float* topk_gate, const int32_t* row_of, const float* zgate, void* out,
                void* stream) {
  return combine_impl(shape, x, y_perm, out_acc, topk_gate, row_of, zgate, out, stream);
}

int moe_pid_init(const moe_shape_t* shape, const float* bias, float* pid_state, void* stream) {
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({bias, pid_state}));
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  return cuda_rc(launch_pid_init(bias, pid_state, shape->n_ffn, as_stream(stream)));
}

int moe_pid_bias_update(const moe_pid_t* pid, const moe_shape_t* shape, const int32_t* counts,
                        const int32_t* nffn_hist, float* bias, float* pid_state, float* stats_out,
                        void* stream) {
  if (!pid) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({counts, nffn_hist, bias, pid_state}));
  MOE_TRY(check_opt({stats_out}));
  if (shape->T == 0) return MOE_ERR_INVALID_ARG;   // frequencies counts / T need T > 0
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  return cuda_rc(launch_pid_update(*pid, counts, nffn_hist, bias, pid_state, stats_out, shape->T,
                                   shape->K, shape->n_ffn, shape->n_ffn + shape->n_zero,
                                   as_stream(stream)));
}

int moe_lb_loss(const moe_shape_t* shape, const float* logits, const int32_t* counts,
                float* prob_mean, float* loss, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({counts, ws}));
  MOE_TRY(check_opt({prob_mean}));
  if (!loss) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0) MOE_TRY(check_ptrs({logits}));
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.scratch_end) return MOE_ERR_WORKSPACE;
  DeviceInfo dev;
  MOE_TRY(current_device_info(&dev));
  return cuda_rc(launch_lb_loss(logits, counts, shape->T, shape->n_ffn + shape->n_zero,
                                shape->n_ffn, shape->K, at<double>(ws, L.lbpart), prob_mean, loss,
                                as_stream(stream)));
}

int moe_forward(const moe_shape_t* shape, const void* x, const float* w_router,
                const float* logits_in, const float* bias, const void* w_gate_up,
                const void* w_down, void* out, int32_t* topk_idx, float* topk_gate,
                int32_t* counts, int32_t* nffn_hist, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({x, bias, w_gate_up, w_down, out, topk_idx, topk_gate, counts, nffn_hist, ws}));
  if (!logits_in) MOE_TRY(check_ptrs({w_router}));
  MOE_TRY(check_opt({logits_in}));
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (shape->T == 0) return MOE_OK;
  const bool fused = shape->combine == MOE_COMBINE_FUSED;
  float* logits = at<float>(ws, L.logits);
  float* zgate = at<float>(ws, L.zgate);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* rowof = at<int32_t>(ws, L.rowof);
  float* rowgate = at<float>(ws, L.rowgate);
  void* xperm = at<char>(ws, L.xperm);
  void* h = at<char>(ws, L.h);
  void* yperm = fused ? nullptr : at<char>(ws, L.yperm);
  float* outacc = fused ? at<float>(ws, L.outacc) : nullptr;
  MOE_TRY(route_impl(shape, x, w_router, nullptr, logits_in, bias, logits, topk_idx, topk_gate,
                     counts, nffn_hist, zgate, ws, ws_bytes, stream));
  MOE_TRY(permute_impl(shape, topk_idx, topk_gate, zgate, x, offsets, perm, rowof, rowgate, xperm,
                       outacc, ws, ws_bytes, stream));
  MOE_TRY(grouped_ffn_impl(shape, x, xperm, offsets, w_gate_up, w_down, perm, rowgate, h, yperm,
                           outacc, nullptr, ws, ws_bytes, stream));
  return combine_impl(shape, x, yperm, outacc, topk_gate, rowof, zgate, out, stream);
}

}  // extern "C"

// ---- end-to-end runs from host memory, overlapped across batches --------------------------
// Batch i's layer kernels run on the caller's stream while batch i+1's input crosses to the
// device on one copy stream and batch i-1's output crosses back on another. Two slots of
// device staging buffers (the caller's) alternate; per slot, "staged" orders the kernels
// after the input copy, "consumed" the next input copy into the slot after the kernels that
// read it, and "drained" the next kernels writing the slot's output after its copy out.
struct moe_host_pipeline {
  moe_shape_t shape;
  int device;
  cudaStream_t compute, h2d, d2h;
  void* x_dev[2];
  float* logits_dev[2];
  void* out_dev[2];
  cudaEvent_t staged[2], consumed[2], drained[2], fork, tail;
  bool used[2];
  bool forked;
  uint64_t n;
};

namespace moe {
namespace {

size_t elt_bytes(const moe_shape_t& s) { return s.dtype == MOE_BF16 ? 2 : 4; }

void destroy_pipeline_parts(moe_host_pipeline* p) {
  for (int b = 0; b < 2; ++b) {
    if (p->staged[b]) cudaEventDestroy(p->staged[b]);
    if (p->consumed[b]) cudaEventDestroy(p->consumed[b]);
    if (p->drained[b]) cudaEventDestroy(p->drained[b]);
  }
  if (p->fork) cudaEventDestroy(p->fork);
  if (p->tail) cudaEventDestroy(p->tail);
  if (p->h2d) cudaStreamDestroy(p->h2d);
  if (p->d2h) cudaStreamDestroy(p->d2h);
  cudaGetLastError();
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_host_pipeline_create(const moe_shape_t* shape, void* const x_dev[2],
                             float* const logits_dev[2], void* const out_dev[2], void* stream,
                             moe_host_pipeline** pipe) {
  using namespace moe;
  if (!pipe || !x_dev || !out_dev) return MOE_ERR_INVALID_ARG;
  *pipe = nullptr;
  MOE_TRY(check_shape(shape));
  MOE_TRY(check_ptrs({x_dev[0], x_dev[1], out_dev[0], out_dev[1]}));
  if (logits_dev) MOE_TRY(check_ptrs({logits_dev[0], logits_dev[1]}));
  DeviceInfo info;
  MOE_TRY(current_device_info(&info));
  moe_host_pipeline* p = static_cast<moe_host_pipeline*>(calloc(1, sizeof(moe_host_pipeline)));
  if (!p) return MOE_ERR_INVALID_ARG;
  p->shape = *shape;
  p->device = info.device;
  p->compute = as_stream(stream);
  for (int b = 0; b < 2; ++b) {
    p->x_dev[b] = x_dev[b];
    p->logits_dev[b] = logits_dev ? logits_dev[b] : nullptr;
    p->out_dev[b] = out_dev[b];
  }
  bool ok = cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p->fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p->tail, cudaEventDisableTiming) == cudaSuccess;
  for (int b = 0; ok && b < 2; ++b)
    ok = cudaEventCreateWithFlags(&p->staged[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->consumed[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->drained[b], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    destroy_pipeline_parts(p);
    free(p);
    return MOE_ERR_CUDA;
  }
  *pipe = p;
  return MOE_OK;
}

int moe_host_pipeline_submit(moe_host_pipeline* p, const void* x_host,
                             const float* logits_in_host, void* out_host, const float* w_router,
                             const float* bias, const void* w_gate_up, const void* w_down,
                             int32_t* topk_idx, float* topk_gate, int32_t* counts,
                             int32_t* nffn_hist, void* ws, size_t ws_bytes) {
  using namespace moe;
  if (!p || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if (logits_in_host && !p->logits_dev[0]) return MOE_ERR_INVALID_ARG;
  const moe_shape_t& s = p->shape;
  // every check moe_forward makes, before anything is queued
  MOE_TRY(check_ptrs({bias, w_gate_up, w_down, topk_idx, topk_gate, counts, nffn_hist, ws}));
  if (!logits_in_host) MOE_TRY(check_ptrs({w_router}));
  if (ws_bytes < layout_of(s).total) return MOE_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) {
    cudaGetLastError();
    return MOE_ERR_INVALID_ARG;
  }
  if (s.T == 0) return MOE_OK;
  const int b = static_cast<int>(p->n & 1);
  const size_t xb = (size_t)s.T * s.H * elt_bytes(s);
  const size_t lb = (size_t)s.T * (s.n_ffn + s.n_zero) * sizeof(float);
  if (!p->forked) {
    // a new sequence starts after the work already on the caller's stream
    MOE_TRY(cuda_rc(cudaEventRecord(p->fork, p->compute)));
    MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->h2d, p->fork, 0)));
    MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->d2h, p->fork, 0)));
    p->forked = true;
  }
  if (p->used[b]) MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->h2d, p->consumed[b], 0)));
  MOE_TRY(cuda_rc(cudaMemcpyAsync(p->x_dev[b], x_host, xb, cudaMemcpyHostToDevice, p->h2d)));
  if (logits_in_host)
    MOE_TRY(cuda_rc(cudaMemcpyAsync(p->logits_dev[b], logits_in_host, lb,
                                    cudaMemcpyHostToDevice, p->h2d)));
  MOE_TRY(cuda_rc(cudaEventRecord(p->staged[b], p->h2d)));
  MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->compute, p->staged[b], 0)));
  if (p->used[b]) MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->compute, p->drained[b], 0)));
  MOE_TRY(moe_forward(&s, p->x_dev[b], w_router, logits_in_host ? p->logits_dev[b] : nullptr,
                      bias, w_gate_up, w_down, p->out_dev[b], topk_idx, topk_gate, counts,
                      nffn_hist, ws, ws_bytes, p->compute));
  MOE_TRY(cuda_rc(cudaEventRecord(p->consumed[b], p->compute)));
  MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->d2h, p->consumed[b], 0)));
  MOE_TRY(cuda_rc(cudaMemcpyAsync(out_host, p->out_dev[b], xb, cudaMemcpyDeviceToHost, p->d2h)));
  MOE_TRY(cuda_rc(cudaEventRecord(p->drained[b], p->d2h)));
  p->used[b] = true;
  ++p->n;
  return MOE_OK;
}

int moe_host_pipeline_join(moe_host_pipeline* p) {
  using namespace moe;
  if (!p) return MOE_ERR_INVALID_ARG;
  MOE_TRY(cuda_rc(cudaEventRecord(p->tail, p->h2d)));
  MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->compute, p->tail, 0)));
  MOE_TRY(cuda_rc(cudaEventRecord(p->tail, p->d2h)));
  MOE_TRY(cuda_rc(cudaStreamWaitEvent(p->compute, p->tail, 0)));
  p->forked = false;
  return MOE_OK;
}

int moe_host_pipeline_destroy(moe_host_pipeline* p) {
  using namespace moe;
  if (!p) return MOE_OK;
  const bool ok = cudaStreamSynchronize(p->h2d) == cudaSuccess &&
                  cudaStreamSynchronize(p->d2h) == cudaSuccess;
  destroy_pipeline_parts(p);
  free(p);
  return ok ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
