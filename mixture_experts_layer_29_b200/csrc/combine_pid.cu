// combine_pid.cu - the combine step and the PID bias update.
//
// Combine (LongCat-Flash Technical Report digest, Key claims, report §2.1: a
// zero-computation expert is an identity map, so it adds g * x; Method: the MoE combine):
//   fused mode          out = out_acc rounded to the output type
//   deterministic mode  out[t] = sum over FFN slots k, in slot order, of s * g_k * y_k,
//                       then + zgate[t] * x[t]; fp32, rounded once.
// PID (report §2.1.1, Fig. 3; zero experts excluded, report §2.1.2): one CTA updates the
// FFN experts' biases from the batch's expert counts and writes the step's statistics.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&q);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(b[i]);
  }
  __device__ static void store(__nv_bfloat16* p, const float (&v)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  __device__ static void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <typename T>
__global__ void __launch_bounds__(256) k_finalize(const float* acc, T* out,
                                                  size_t n) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int V = Vec<T>::N;
  const size_t nv = n / V;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv;
       i += (size_t)gridDim.x * blockDim.x) {
    float v[V];
#pragma unroll
    for (int j = 0; j < V; j += 4) {
      const float4 q = reinterpret_cast<const float4*>(acc)[i * (V / 4) + j / 4];
      v[j] = q.x; v[j + 1] = q.y; v[j + 2] = q.z; v[j + 3] = q.w;
    }
    Vec<T>::store(out + i * V, v);
  }
}

// G rows are loaded before they are summed: G = 4 for small batches (more loads in
// flight per thread), 1 for large ones (fewer registers, more CTAs per SM).
template <typename T, int G>
__global__ void __launch_bounds__(256) k_combine_det(const T* x, const T* y_perm,
                                                     const float* topk_gate,
                                                     const int32_t* row_of,
                                                     const float* zgate,
                                                     T* out, int H, int K, float scale) {
  constexpr int V = Vec<T>::N;
  __shared__ int s_row[32 + G];
  __shared__ float s_g[32 + G];
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  if (threadIdx.x < 32 + G) {
    const bool in = threadIdx.x < K;
    s_row[threadIdx.x] = in ? row_of[(size_t)t * K + threadIdx.x] : -1;
    s_g[threadIdx.x] = in ? scale * topk_gate[(size_t)t * K + threadIdx.x] : 0.f;
  }
  __syncthreads();
  const float zg = zgate[t];
  // blockIdx.y picks a contiguous slice of the columns (several blocks per token when T
  // is small)
  const int per = (H / V + gridDim.y - 1) / gridDim.y * V;
  const int c_end = min(H, (int)(blockIdx.y + 1) * per);
  for (int c = blockIdx.y * per + threadIdx.x * V; c < c_end; c += blockDim.x * V) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    // slots in order
    for (int k0 = 0; k0 < K; k0 += G) {
      float y[G][V];
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const int r = s_row[k0 + u];
        if (r >= 0) Vec<T>::load(y_perm + (size_t)r * H + c, y[u]);
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        if (s_row[k0 + u] < 0) continue;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(s_g[k0 + u], y[u][i], acc[i]);
      }
    }
    float xv[V];
    Vec<T>::load(x + (size_t)t * H + c, xv);
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = fmaf(zg, xv[i], acc[i]);
    Vec<T>::store(out + (size_t)t * H + c, acc);
  }
}

__global__ void k_pid_init(const float* bias, float* st, int n_ffn) {
  pdl_launch_dependents();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_ffn; i += gridDim.x * blockDim.x) {
    st[i] = bias[i];
    st[n_ffn + i] = 0.f;
    st[2 * n_ffn + i] = 0.f;
  }
}

// One CTA of kPidThreads; thread i updates experts i, i + kPidThreads, ... (each expert's
// bias in fp32, in the fixed order of the PID law). The statistics are reduced in one
// pass: warp butterflies, then warp 0 over the warps (fixed order).
constexpr int kPidThreads = 256;

__global__ void __launch_bounds__(kPidThreads) k_pid_update(moe_pid_t pid,
                                                            const int32_t* counts,
                                                            const int32_t* hist,
                                                            float* bias,
                                                            float* st,
                                                            float* stats, int T,
                                                            int K, int n_ffn, int E) {
  constexpr int W = kPidThreads / 32;
  __shared__ double red[W][8];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // v: [0] FFN count, [1] max FFN count, [2] FFN experts hit, [3] zero-expert count,
  //    [4] |e|, [5] max |e|, [6] n * hist[n], [7] n^2 * hist[n]
  double v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const float tau = __fdiv_rn(__fmul_rn(pid.target_ratio, (float)K), (float)n_ffn);
  for (int i = tid; i < n_ffn; i += kPidThreads) {
    const int c = counts[i];
    const float f = __fdiv_rn((float)c, (float)T);
    const float e = __fsub_rn(tau, f);
    const float integ = __fadd_rn(st[n_ffn + i], e);
    const float deriv = __fsub_rn(e, st[2 * n_ffn + i]);
    float b = __fadd_rn(st[i], __fmul_rn(pid.kp, e));
    b = __fadd_rn(b, __fmul_rn(pid.ki, integ));
    b = __fadd_rn(b, __fmul_rn(pid.kd, deriv));
    bias[i] = b;
    st[n_ffn + i] = integ;
    st[2 * n_ffn + i] = e;
    v[0] += (double)c;
    v[1] = fmax(v[1], (double)c);
    v[2] += c > 0 ? 1.0 : 0.0;
    v[4] += fabs((double)e);
    v[5] = fmax(v[5], fabs((double)e));
  }
  for (int j = n_ffn + tid; j < E; j += kPidThreads) v[3] += (double)counts[j];
  for (int n = tid; n <= K; n += kPidThreads) {
    v[6] += (double)hist[n] * n;
    v[7] += (double)hist[n] * n * n;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const double u = __shfl_xor_sync(0xffffffffu, v[k], o);
      v[k] = (k == 1 || k == 5) ? fmax(v[k], u) : v[k] + u;
    }
  }
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 8; ++k) red[warp][k] = v[k];
  __syncthreads();
  if (stats && warp == 0) {
    // lane k < 8 combines statistic k over the warps in order
    double r = 0.0;
    if (lane < 8) {
      const bool mx = lane == 1 || lane == 5;
      for (int w = 0; w < W; ++w) r = mx ? fmax(r, red[w][lane]) : r + red[w][lane];
    }
    double rr[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) rr[k] = __shfl_sync(0xffffffffu, r, k);
    if (lane == 0) {
      const double mean = rr[6] / T;
      const double var = fmax(0.0, rr[7] / T - mean * mean);
      const double mean_load = rr[0] / n_ffn;
      stats[0] = (float)(mean / K);
      stats[1] = (float)mean;
      stats[2] = (float)sqrt(var);
      stats[3] = (float)(mean_load > 0.0 ? rr[1] / mean_load : 0.0);
      stats[4] = (float)rr[2];
      stats[5] = (float)(rr[3] / ((double)T * K));
      stats[6] = (float)(rr[4] / n_ffn);
      stats[7] = (float)rr[5];
    }
  }
}

}  // namespace

cudaError_t launch_finalize(const float* out_acc, void* out, int out_is_bf16, size_t n,
                            cudaStream_t st) {
  const size_t work = n / 8;
  int blocks = (int)((work + 255) / 256);
  if (blocks > 8192) blocks = 8192;
  if (blocks < 1) blocks = 1;
  const cudaError_t e =
      out_is_bf16 ? launch_kernel(k_finalize<__nv_bfloat16>, blocks, 256, 0, st, 1, out_acc,
                                  static_cast<__nv_bfloat16*>(out), n)
                  : launch_kernel(k_finalize<float>, blocks, 256, 0, st, 1, out_acc,
                                  static_cast<float*>(out), n);
  count_launch();
  return e;
}

cudaError_t launch_combine_det(const void* x, const void* y_perm, const float* topk_gate,
                               const int32_t* row_of, const float* zgate, void* out,
                               int is_bf16, int T, int H, int K, float scale, cudaStream_t st) {
  // enough blocks for every SM even at small T (one CTA per token and column slice)
  const int V = is_bf16 ? 8 : 4;
  int nseg = (2 * 148 + T - 1) / T;
  const int max_seg = (H / V + 255) / 256;
  if (nseg > max_seg) nseg = max_seg;
  if (nseg < 1) nseg = 1;
  const dim3 grid(T, nseg);
  const bool small = T < 1024;
  const cudaError_t e =
      is_bf16 ? launch_kernel(small ? k_combine_det<__nv_bfloat16, 4> : k_combine_det<__nv_bfloat16, 1>,
                              grid, 256, 0, st, 1, static_cast<const __nv_bfloat16*>(x),
                              static_cast<const __nv_bfloat16*>(y_perm), topk_gate, row_of, zgate,
                              static_cast<__nv_bfloat16*>(out), H, K, scale)
              : launch_kernel(small ? k_combine_det<float, 4> : k_combine_det<float, 1>, grid, 256,
                              0, st, 1, static_cast<const float*>(x),
                              static_cast<const float*>(y_perm), topk_gate, row_of, zgate,
                              static_cast<float*>(out), H, K, scale);
  count_launch();
  return e;
}

cudaError_t launch_pid_init(const float* bias, float* pid_state, int n_ffn, cudaStream_t st) {
  const cudaError_t e = launch_kernel(k_pid_init, (n_ffn + 255) / 256, 256, 0, st, 1, bias,
                                      pid_state, n_ffn);
  count_launch();
  return e;
}

cudaError_t launch_pid_update(const moe_pid_t& pid, const int32_t* counts,
                              const int32_t* nffn_hist, float* bias, float* pid_state,
                              float* stats, int T, int K, int n_ffn, int E, cudaStream_t st) {
  const cudaError_t e = launch_kernel(k_pid_update, 1, kPidThreads, 0, st, 1, pid, counts, nffn_hist,
                                      bias, pid_state, stats, T, K, n_ffn, E);
  count_launch();
  return e;
}

}  // namespace moe
