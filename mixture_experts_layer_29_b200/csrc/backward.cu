// backward.cu - the layer's backward outside the expert GEMMs (those are in gemm_bwd.cu).
//
// The forward, differentiated with the expert selection held fixed (it is piecewise
// constant in the inputs) and no gradient to the selection bias (LongCat-Flash Technical
// Report digest, Key claims, report §2.1.1: the bias only steers selection and is set by the
// PID controller):
//   out[t] = sum over FFN picks of s g_k y_k(x_t) + sum over zero picks of g_k x_t,
//   g_k = p[t, e_k],  p = softmax(x_t W_r^T)
// Kernels:
//   k_bwd_dy_dgate   per token: dy[r] = s g_k dout_t on each FFN row r (bf16), and each
//                    pick's gate gradient: s <dout_t, y_r> (FFN) or <dout_t, x_t> (zero)
//   k_bwd_router     per token: p again from the logits (double), dp at the picks,
//                    dL = p * (dp - <p, dp>), split exactly into three bf16 parts
//                    (hi = bf16(dL), mid = bf16(dL - hi), lo = dL - hi - mid) for the
//                    router's tensor-core GEMMs in gemm_bwd.cu: d_router = dL^T x (all
//                    three parts: exact products, fp32 sums) and dx = dL W_r (hi parts)
//   k_to_bf16        W_r in bf16 for the latter
//   k_bwd_dx_combine dx[t] += sum over FFN slots (in order) of dx_perm[row] + zgate_t dout_t
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&q);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(b[i]);
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kTok = 256;   // threads per token CTA

// One CTA per token; thread i owns columns 8i, 8i + 8 kTok, ... of the row. G slots' rows
// are loaded before they are used (more loads in flight per thread).
template <int G>
__global__ void __launch_bounds__(kTok) k_bwd_dy_dgate(
    const __nv_bfloat16* dout, const __nv_bfloat16* x,
    const __nv_bfloat16* y_perm, const int32_t* topk_idx,
    const float* topk_gate, const int32_t* row_of, int H, int K,
    int n_ffn, float scale, __nv_bfloat16* dy, float* d_gate) {
  __shared__ int s_row[32];
  __shared__ float s_g[32];
  __shared__ float s_red[kTok / 32][33];
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 32) {
    const bool in = threadIdx.x < K;
    const int e = in ? topk_idx[(size_t)t * K + threadIdx.x] : 0;
    s_row[threadIdx.x] = in && e < n_ffn ? row_of[(size_t)t * K + threadIdx.x] : -1;
    s_g[threadIdx.x] = in ? topk_gate[(size_t)t * K + threadIdx.x] : 0.f;
  }
  __syncthreads();
  float dot[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) dot[k] = 0.f;
  for (int c = threadIdx.x * 8; c < H; c += kTok * 8) {
    float d[8], xv[8];
    load8(dout + (size_t)t * H + c, d);
    load8(x + (size_t)t * H + c, xv);
#pragma unroll
    for (int k0 = 0; k0 < 32; k0 += G) {
      if (k0 >= K) break;
      float y[G][8];
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const int r = s_row[k0 + u];
        if (k0 + u < K && r >= 0) load8(y_perm + (size_t)r * H + c, y[u]);
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const int k = k0 + u;
        if (k >= K) break;
        const int r = s_row[k];
        if (r >= 0) {
          const float gs = scale * s_g[k];
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(gs * d[2 * i], gs * d[2 * i + 1]);
          *reinterpret_cast<uint4*>(dy + (size_t)r * H + c) = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
          for (int i = 0; i < 8; ++i) dot[k] = fmaf(d[i], y[u][i], dot[k]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) dot[k] = fmaf(d[i], xv[i], dot[k]);
        }
      }
    }
  }
  // block sums of the K dot products (fixed order)
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    if (k >= K) break;
    float v = dot[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_red[warp][k] = v;
  }
  __syncthreads();
  if (threadIdx.x < K) {
    float v = 0.f;
    for (int w = 0; w < kTok / 32; ++w) v += s_red[w][threadIdx.x];
    d_gate[(size_t)t * K + threadIdx.x] = s_row[threadIdx.x] >= 0 ? scale * v : v;
  }
}

// One warp per token: dL[t, e] = p_e (dp_e - sum_k p_{e_k} dg_k), dp_e = dg_k at e = e_k.
// dl3: [3][Tp][E] bf16, part p of token t at row p Tp + t; rows [T, Tp) of every part are
// written as zeros. Block 0 also writes the two one-group offset tables of the router
// GEMMs: offs_k = {0, 3 Tp}, offs_m = {0, T}.
template <int J>
__global__ void __launch_bounds__(256) k_bwd_router(const float* logits,
                                                    const int32_t* topk_idx,
                                                    const float* d_gate, int T,
                                                    int Tp, int E, int K,
                                                    __nv_bfloat16* dl3,
                                                    int32_t* offs) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    offs[0] = 0;
    offs[1] = 3 * Tp;
    offs[2] = 0;
    offs[3] = T;
  }
  if (t >= Tp) return;
  if (t >= T) {
    for (int e = lane; e < E; e += 32)
      for (int p = 0; p < 3; ++p) dl3[((size_t)p * Tp + t) * E + e] = __float2bfloat16_rn(0.f);
    return;
  }
  const float* Lr = logits + (size_t)t * E;
  float lv[J];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    lv[j] = e < E ? Lr[e] : -INFINITY;
    m = fmaxf(m, lv[j]);
  }
  m = warp_max(m);
  double ex[J], sum = 0.0;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    ex[j] = e < E ? exp((double)lv[j] - (double)m) : 0.0;
    sum += ex[j];
  }
  sum = warp_sum(sum);
  const double inv = 1.0 / sum;
  // the picks: lane k < K holds (e_k, dg_k)
  const int my_e = lane < K ? topk_idx[(size_t)t * K + lane] : -1;
  const float my_dg = lane < K ? d_gate[(size_t)t * K + lane] : 0.f;
  double dpe[J];
#pragma unroll
  for (int j = 0; j < J; ++j) dpe[j] = 0.0;
  double dot = 0.0;
  for (int k = 0; k < K; ++k) {
    const int ek = __shfl_sync(0xffffffffu, my_e, k);
    const float dgk = __shfl_sync(0xffffffffu, my_dg, k);
#pragma unroll
    for (int j = 0; j < J; ++j)
      if (ek == lane + 32 * j) {
        dpe[j] = dgk;
        dot += ex[j] * inv * (double)dgk;
      }
  }
  dot = warp_sum(dot);
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      const float v = (float)(ex[j] * inv * (dpe[j] - dot));
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const float r1 = __fsub_rn(v, __bfloat162float(hi));
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(r1, __bfloat162float(mid)));
      dl3[(size_t)t * E + e] = hi;
      dl3[((size_t)Tp + t) * E + e] = mid;
      dl3[(2 * (size_t)Tp + t) * E + e] = lo;
    }
  }
}

__global__ void __launch_bounds__(256) k_to_bf16(const float* a,
                                                 __nv_bfloat16* out, size_t n) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(a[i]);
}

// dx[t] += sum over FFN slots k (in order) of dx_perm[row_of[t, k]] + zgate_t * dout_t
__global__ void __launch_bounds__(kTok) k_bwd_dx_combine(
    const float* dx_perm, const __nv_bfloat16* dout,
    const int32_t* topk_idx, const float* topk_gate,
    const int32_t* row_of, int H, int K, int n_ffn, float* dx) {
  __shared__ int s_row[32];
  __shared__ float s_z;
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  if (threadIdx.x < 32) {
    const int k = threadIdx.x;
    int r = -1;
    float zg = 0.f;
    if (k < K) {
      const int e = topk_idx[(size_t)t * K + k];
      if (e < n_ffn) r = row_of[(size_t)t * K + k];
      else zg = topk_gate[(size_t)t * K + k];
    }
    s_row[k] = r;
    // zgate in slot order (lane 0 adds the lanes' terms one by one)
    float z = 0.f;
    for (int j = 0; j < K; ++j) z += __shfl_sync(0xffffffffu, zg, j);
    if (k == 0) s_z = z;
  }
  __syncthreads();
  const float z = s_z;
  for (int c = threadIdx.x * 8; c < H; c += kTok * 8) {
    float acc[8], d[8];
    load8(dx + (size_t)t * H + c, acc);
    for (int k = 0; k < K; ++k) {
      const int r = s_row[k];
      if (r < 0) continue;
      float v[8];
      load8(dx_perm + (size_t)r * H + c, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
    load8(dout + (size_t)t * H + c, d);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(z, d[i], acc[i]);
    *reinterpret_cast<float4*>(dx + (size_t)t * H + c) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(dx + (size_t)t * H + c + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

cudaError_t launch_bwd_dy_dgate(const void* dout, const void* x, const void* y_perm,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* row_of, int T, int H, int K, int n_ffn,
                                float scale, void* dy, float* d_gate, cudaStream_t st) {
  const cudaError_t e = launch_kernel(
      tuning(MOE_TUNE_BWD_DY_ROWS) == 1 ? k_bwd_dy_dgate<1> : k_bwd_dy_dgate<4>, T, kTok, 0, st, 1,
      static_cast<const __nv_bfloat16*>(dout),
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y_perm), topk_idx,
      topk_gate, row_of, H, K, n_ffn, scale, static_cast<__nv_bfloat16*>(dy), d_gate);
  count_launch();
  return e;
}

cudaError_t launch_bwd_router(const float* logits, const int32_t* topk_idx, const float* d_gate,
                              int T, int Tp, int E, int K, void* dl3, int32_t* offs,
                              const float* w_router, void* wr16, int H, cudaStream_t st) {
  const int J = (E + 31) / 32;
  const int blocks = (Tp + 7) / 8;
  cudaError_t e = cudaErrorInvalidValue;
#define MOE_BR_CASE(JJ)                                                                    \
  if (J <= JJ) {                                                                           \
    e = launch_kernel(k_bwd_router<JJ>, blocks, 256, 0, st, 1, logits, topk_idx, d_gate, T, \
                      Tp, E, K, static_cast<__nv_bfloat16*>(dl3), offs);                  \
  } else
  MOE_BR_CASE(4) MOE_BR_CASE(8) MOE_BR_CASE(16) MOE_BR_CASE(24) MOE_BR_CASE(32) {
    return cudaErrorInvalidValue;
  }
#undef MOE_BR_CASE
  count_launch();
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)E * H;
  int cb = (int)((n + 255) / 256);
  if (cb > 4096) cb = 4096;
  e = launch_kernel(k_to_bf16, cb, 256, 0, st, 1, w_router, static_cast<__nv_bfloat16*>(wr16), n);
  count_launch();
  return e;
}

cudaError_t launch_bwd_dx_combine(const float* dx_perm, const void* dout, const int32_t* topk_idx,
                                  const float* topk_gate, const int32_t* row_of, int T, int H,
                                  int K, int n_ffn, float* dx, cudaStream_t st) {
  const cudaError_t e =
      launch_kernel(k_bwd_dx_combine, T, kTok, 0, st, 1, dx_perm,
                    static_cast<const __nv_bfloat16*>(dout), topk_idx, topk_gate, row_of, H, K,
                    n_ffn, dx);
  count_launch();
  return e;
}

}  // namespace moe
