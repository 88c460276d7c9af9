// lbloss.cu - the device-level load-balance loss of one batch (forward value).
//
// LongCat-Flash Technical Report digest, Key claims, report §2.1.1 / §2.1.2 Eqs. 3-5: the
// zero-computation experts' share is held by a device-level load-balance loss, DeepSeek-V3's
// balance loss extended so that all zero-computation experts form one virtual group. The
// equations are not printed; the form computed here is
//   f_i = E c_i / (K T)                    c_i: tokens that picked expert i
//   P_i = (1/T) sum_t p[t, i]              p: the router softmax over all E experts
//   L   = sum_{i < N} f_i P_i + mean_{i >= N}(f_i) * sum_{i >= N} P_i
// (one group per FFN expert, one group of every zero expert; a balanced batch gives 1).
//
// k_lb_partial: CTA c sums p over tokens [64c, 64c + 64) for every expert, in double and in
//               a fixed order (warp w takes 16 tokens in order; the warps are added in
//               order), into part[c][E].
// k_lb_finish:  one CTA: P_i = (sum over c in order of part[c][i]) / T, then the loss with
//               fixed-order block reductions. Both kernels are deterministic.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kLbWarps = 4;
constexpr int kLbTokens = 64;                        // tokens per CTA
constexpr int kLbPerWarp = kLbTokens / kLbWarps;

template <int J>
__global__ void __launch_bounds__(kLbWarps * 32) k_lb_partial(const float* logits,
                                                             int T, int E,
                                                             double* part) {
  __shared__ double s_acc[kLbWarps][32 * J];
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double acc[J];
#pragma unroll
  for (int j = 0; j < J; ++j) acc[j] = 0.0;
  const int t0 = blockIdx.x * kLbTokens + warp * kLbPerWarp;
  for (int i = 0; i < kLbPerWarp; ++i) {
    const int t = t0 + i;
    if (t >= T) break;                               // warp-uniform
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
    const double dm = (double)m;
    double ex[J];
    double sum = 0.0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      ex[j] = e < E ? exp((double)lv[j] - dm) : 0.0;
      sum += ex[j];
    }
    sum = warp_sum(sum);
    const double inv = 1.0 / sum;
#pragma unroll
    for (int j = 0; j < J; ++j) acc[j] += ex[j] * inv;
  }
#pragma unroll
  for (int j = 0; j < J; ++j) s_acc[warp][lane + 32 * j] = acc[j];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double v = s_acc[0][e];
#pragma unroll
    for (int w = 1; w < kLbWarps; ++w) v += s_acc[w][e];
    part[(size_t)blockIdx.x * E + e] = v;
  }
}

// block-wide sum of one double per thread, fixed order (warp butterflies, then warps in
// order by thread 0); every thread gets the result
__device__ __forceinline__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += red[w];
    red[32] = r;
  }
  __syncthreads();
  return red[32];
}

__global__ void __launch_bounds__(1024) k_lb_finish(const double* part, int nchunk,
                                                    const int32_t* counts, int T,
                                                    int E, int n_ffn, int K,
                                                    float* prob_mean,
                                                    float* loss) {
  __shared__ double red[33];
  pdl_launch_dependents();
  pdl_wait();
  const int e = threadIdx.x;
  double P = 0.0, f = 0.0;
  if (e < E && T > 0) {
    for (int c = 0; c < nchunk; ++c) P += part[(size_t)c * E + e];
    P /= (double)T;
    f = (double)E * (double)counts[e] / ((double)K * (double)T);
  }
  if (e < E && prob_mean) prob_mean[e] = (float)P;
  const bool ffn = e < n_ffn, zero = e >= n_ffn && e < E;
  const double ffn_term = block_sum(ffn ? f * P : 0.0, red);
  const double zero_f = block_sum(zero ? f : 0.0, red);
  const double zero_P = block_sum(zero ? P : 0.0, red);
  if (threadIdx.x == 0) {
    const int n_zero = E - n_ffn;
    const double l = ffn_term + (n_zero > 0 ? zero_f / n_zero * zero_P : 0.0);
    loss[0] = (float)l;
  }
}

template <int J>
cudaError_t launch_lb_j(const float* logits, int T, int E, double* part, cudaStream_t st) {
  const int nchunk = (T + kLbTokens - 1) / kLbTokens;
  return launch_kernel(k_lb_partial<J>, nchunk, kLbWarps * 32, 0, st, 1, logits, T, E, part);
}

}  // namespace

size_t lb_partial_bytes(int T, int E) {
  return (size_t)((T + kLbTokens - 1) / kLbTokens) * E * sizeof(double);
}

cudaError_t launch_lb_loss(const float* logits, const int32_t* counts, int T, int E, int n_ffn,
                           int K, double* part, float* prob_mean, float* loss, cudaStream_t st) {
  cudaError_t err = cudaSuccess;
  if (T > 0) {
    const int J = (E + 31) / 32;
#define MOE_LB_CASE(JJ) \
  if (J <= JJ) {        \
    err = launch_lb_j<JJ>(logits, T, E, part, st); \
  } else
    MOE_LB_CASE(4) MOE_LB_CASE(8) MOE_LB_CASE(16) MOE_LB_CASE(24) MOE_LB_CASE(32) {
      return cudaErrorInvalidValue;
    }
#undef MOE_LB_CASE
    count_launch();
    if (err != cudaSuccess) return err;
  }
  const int nchunk = (T + kLbTokens - 1) / kLbTokens;
  err = launch_kernel(k_lb_finish, 1, 1024, 0, st, 1, part, nchunk, counts, T, E, n_ffn, K,
                      prob_mean, loss);
  count_launch();
  return err;
}

}  // namespace moe
