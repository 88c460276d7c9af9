// router.cu - router logits (fp32 GEMM on the CUDA cores) and the warp-per-token softmax,
// bias-adjusted top-K and expert histogram.
//
// LongCat-Flash Technical Report digest, Key claims (report §2.1, §2.4): the router picks
// K experts per token from the combined pool of FFN and zero-computation experts; (report
// §2.1.1) a per-expert bias steers the selection, the gates stay the softmax values.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

// ---------------------------------------------------------------------------------------
// logits[t, e] = sum_h x[t, h] * w_router[e, h]   (fp32 FMA, smem-tiled, optional split-K)
// 128 x 128 output tile per CTA, 16-deep k slices, 256 threads with an 8 x 8 micro-tile.
// Split-K writes fp32 partials that a second kernel sums in split order, so the logits
// are bit-reproducible.
// ---------------------------------------------------------------------------------------
namespace {
constexpr int RB = 128, RK = 16, RPAD = 4;
constexpr int kSmMax = 160;   // sizing bound for the split-K partial buffer

template <bool XBF16>
__device__ __forceinline__ void load_x_slice(const void* x, int T, int H, int row0, int k0,
                                             float (&v)[8], int& r, int& kk) {
  const int tid = threadIdx.x;
  if (XBF16) {
    r = tid >> 1;
    kk = (tid & 1) * 8;
    const int t = row0 + r;
    if (t < T) {
      const uint4 q = *reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(x) + (size_t)t * H + k0 + kk);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&q);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(b[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
  } else {
    // two float4 per thread: rows tid/4 and tid/4 + 64, k quarter tid%4
    r = tid >> 2;
    kk = (tid & 3) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = row0 + r + 64 * h;
      float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < T) q = *reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * H + k0 + kk);
      v[4 * h + 0] = q.x; v[4 * h + 1] = q.y; v[4 * h + 2] = q.z; v[4 * h + 3] = q.w;
    }
  }
}

__device__ __forceinline__ void load_w_slice(const float* __restrict__ w, int E, int H, int col0, int k0,
                                             float (&v)[8]) {
  const int tid = threadIdx.x;
  const int r = tid >> 2, kk = (tid & 3) * 4;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e = col0 + r + 64 * h;
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < E) q = *reinterpret_cast<const float4*>(w + (size_t)e * H + k0 + kk);
    v[4 * h + 0] = q.x; v[4 * h + 1] = q.y; v[4 * h + 2] = q.z; v[4 * h + 3] = q.w;
  }
}

template <bool XBF16>
__global__ void __launch_bounds__(256, 2) k_router_logits(const void* x,
                                                       const float* __restrict__ w, int T, int E,
                                                       int H, int kchunk, float* out,
                                                       size_t split_stride, ZeroSpec zero) {
  __shared__ __align__(16) float As[2][RK][RB + RPAD];
  __shared__ __align__(16) float Bs[2][RK][RB + RPAD];
  pdl_launch_dependents();
  pdl_wait();
  zero.run(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z),
           gridDim.x * gridDim.y * gridDim.z, threadIdx.x, blockDim.x);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int row0 = blockIdx.y * RB, col0 = blockIdx.x * RB;
  const int kbeg = blockIdx.z * kchunk;
  const int kend = min(H, kbeg + kchunk);

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  float xa[8], wb[8];
  int xr, xk;
  auto stash = [&](int buf) {
    if (XBF16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) As[buf][xk + i][xr] = xa[i];
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) As[buf][xk + i][xr + 64 * h] = xa[4 * h + i];
    }
    const int wr = tid >> 2, wk = (tid & 3) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) Bs[buf][wk + i][wr + 64 * h] = wb[4 * h + i];
  };

  int buf = 0;
  if (kbeg < kend) {
    load_x_slice<XBF16>(x, T, H, row0, kbeg, xa, xr, xk);
    load_w_slice(w, E, H, col0, kbeg, wb);
    stash(0);
  }
  __syncthreads();
  for (int k0 = kbeg; k0 < kend; k0 += RK) {
    const bool more = k0 + RK < kend;
    if (more) {
      load_x_slice<XBF16>(x, T, H, row0, k0 + RK, xa, xr, xk);
      load_w_slice(w, E, H, col0, k0 + RK, wb);
    }
#pragma unroll
    for (int kk = 0; kk < RK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }

  float* dst = out + blockIdx.z * split_stride;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = row0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = col0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (e < E) dst[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// logits = sum over splits s = 0, 1, ... of partial[s] (fixed order)
__global__ void k_router_splitk_sum(const float* partial, int S, size_t n,
                                    float* logits) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float a = partial[i];
    for (int s = 1; s < S; ++s) a += partial[s * n + i];
    logits[i] = a;
  }
}
}  // namespace

cudaError_t launch_splitk_sum(const float* partial, int S, size_t n, float* out, cudaStream_t st) {
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  const cudaError_t e = launch_kernel(k_router_splitk_sum, blocks, 256, 0, st, 1, partial, S, n, out);
  count_launch();
  return e;
}

int router_splitk(int T, int E, int H, int sm_count) {
  if (sm_count > kSmMax) sm_count = kSmMax;
  const long tiles = (long)((T + RB - 1) / RB) * ((E + RB - 1) / RB);
  if (tiles <= 0 || tiles >= sm_count) return 1;
  long s = (2L * sm_count + tiles - 1) / tiles;
  const long smax = H / 64 > 0 ? H / 64 : 1;     // at least 64 of H per split
  if (s > smax) s = smax;
  if (s > 32) s = 32;
  if (s < 1) s = 1;
  // the effective split count: slices of a multiple of RK, none empty
  int kchunk = (H + (int)s - 1) / (int)s;
  kchunk = (kchunk + RK - 1) / RK * RK;
  return (H + kchunk - 1) / kchunk;
}

size_t router_partial_bytes(int T, int E, int H, int sm_count_max) {
  const int s = router_splitk(T, E, H, sm_count_max > 0 ? sm_count_max : kSmMax);
  return s > 1 ? (size_t)s * T * E * sizeof(float) : 0;
}

cudaError_t launch_router_logits(const void* x, int x_is_bf16, const float* w_router, int T,
                                 int E, int H, float* logits, float* partial, int splitk,
                                 ZeroSpec zero, cudaStream_t st) {
  int kchunk = (H + splitk - 1) / splitk;
  kchunk = (kchunk + RK - 1) / RK * RK;
  const int S = (H + kchunk - 1) / kchunk;
  dim3 grid((E + RB - 1) / RB, (T + RB - 1) / RB, S);
  float* dst = S > 1 ? partial : logits;
  const size_t stride = (size_t)T * E;
  const cudaError_t e = launch_kernel(x_is_bf16 ? k_router_logits<true> : k_router_logits<false>,
                                      grid, 256, 0, st, 1, x, w_router, T, E, H, kchunk, dst,
                                      stride, zero);
  count_launch();
  // with S > 1 the partials are summed in split order (by the top-K kernel or a sum kernel)
  return e;
}

// ---------------------------------------------------------------------------------------
// Softmax + bias-adjusted top-K, one warp per token.
// Lane l holds experts l, l + 32, ... (J groups). exp(L - max) is evaluated in fp32 on
// the exactly split argument (hi + lo, exp(hi) * (1 + lo)), summed in double, and
// normalised with a double reciprocal, so p is within a few fp32 ulps of the float64
// softmax. The selection score is the fp32 sum p + b (a zero result stored as +0); the K
// picks are the first K experts in the order (score descending, expert index ascending).
//
// Selection: theta = the K-th largest of the 32 lane maxima. At least K scores are >=
// theta, so every pick has a score >= theta; the candidates (scores >= theta, typically
// 12 to 25 of 768) are packed into shared memory and each candidate's rank in the order
// above is counted directly. Should more than 32 candidates pass (many equal scores),
// K rounds of a warp-wide argmax over all experts take over. Both give the same picks.
// Counts and the FFN-pick histogram go through shared memory (8-warp CTAs) or straight
// to global integer atomics (one-warp CTAs), with the token's zero-expert gate sum.
// ---------------------------------------------------------------------------------------
namespace {

// exp(d) for d = L - max given exactly in double, evaluated as exp(hi) * (1 + lo)
__device__ __forceinline__ float exp_split(float L, double dm) {
  const double d = (double)L - dm;
  const float dh = (float)d;
  const float dl = (float)(d - (double)dh);
  const float v = expf(dh);
  return fmaf(v, dl, v);
}

struct WarpScratch {        // per warp, in shared memory
  float cs[32];             // candidate scores
  int ce[32];               // candidate experts
  float cp[32];             // candidate gates
  int se[32];               // picks by rank
  float sp[32];
};

// lv[j] holds the logit of expert lane + 32 j (-inf past E). Writes the picks of token t
// and adds them to cnt / hist (shared or global memory).
template <int J>
__device__ __forceinline__ void route_token(float (&lv)[J], const float (&bia)[J], int lane, int t,
                                            int E, int n_ffn, int K, WarpScratch& ws,
                                            int32_t* topk_idx,
                                            float* topk_gate,
                                            float* zgate, int* cnt, int* hist) {
  constexpr unsigned kFull = 0xffffffffu;
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < J; ++j) m = fmaxf(m, lv[j]);
  m = warp_max(m);
  const double dm = (double)m;
  double sum = 0.0;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    const float v = e < E ? exp_split(lv[j], dm) : 0.f;
    lv[j] = v;                                       // lv now holds exp(L - max)
    sum += (double)v;
  }
  sum = warp_sum(sum);
  const double inv = 1.0 / sum;
  float p[J], sc[J];
  float lm = -INFINITY;                              // this lane's largest score
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    p[j] = (float)((double)lv[j] * inv);
    float v = __fadd_rn(p[j], bia[j]);
    if (v == 0.0f) v = 0.0f;                          // -0 -> +0
    sc[j] = e < E ? v : -INFINITY;
    lm = fmaxf(lm, sc[j]);
  }
  // theta: the K-th largest lane maximum (rank by value descending, lane ascending)
  int rk = 0;
#pragma unroll
  for (int i = 1; i < 32; ++i) {
    const int src = (lane + i) & 31;
    const float o = __shfl_sync(kFull, lm, src);
    rk += (o > lm || (o == lm && src < lane)) ? 1 : 0;
  }
  const float theta = __shfl_sync(kFull, lm, __ffs(__ballot_sync(kFull, rk == K - 1)) - 1);
  uint32_t cm = 0u;
#pragma unroll
  for (int j = 0; j < J; ++j)
    if (sc[j] >= theta) cm |= 1u << j;
  const int cnt_l = __popc(cm);
  const int incl = warp_inclusive_scan(cnt_l);
  const int total = __shfl_sync(kFull, incl, 31);
  int my_e = 0;
  float my_g = 0.f;
  if (total <= 32) {
    int pos = incl - cnt_l;
#pragma unroll
    for (int j = 0; j < J; ++j)
      if ((cm >> j) & 1u) {
        ws.cs[pos] = sc[j];
        ws.ce[pos] = lane + 32 * j;
        ws.cp[pos] = p[j];
        ++pos;
      }
    __syncwarp();
    float cs = 0.f;
    int ce = 0;
    int r = 0;
    if (lane < total) {
      cs = ws.cs[lane];
      ce = ws.ce[lane];
#pragma unroll 4
      for (int i = 0; i < total; ++i) {
        const float os = ws.cs[i];
        const int oe = ws.ce[i];
        r += (os > cs || (os == cs && oe < ce)) ? 1 : 0;
      }
      if (r < K) {
        ws.se[r] = ce;
        ws.sp[r] = ws.cp[lane];
      }
    }
    __syncwarp();
    if (lane < K) {
      my_e = ws.se[lane];
      my_g = ws.sp[lane];
    }
    __syncwarp();
  } else {
    // K rounds of a warp argmax on (score descending, expert index ascending)
    uint32_t taken = 0u;
    for (int k = 0; k < K; ++k) {
      float bs = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((taken >> j) & 1u) && (sc[j] > bs || be == 0x7fffffff)) {
          bs = sc[j];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(kFull, bs, o);
        const int oe = __shfl_xor_sync(kFull, be, o);
        if (os > bs || (os == bs && oe < be)) {
          bs = os;
          be = oe;
        }
      }
      const int owner = be & 31, jw = be >> 5;
      float g = 0.f;
#pragma unroll
      for (int j = 0; j < J; ++j)
        if (j == jw) g = p[j];
      if (lane == owner) taken |= 1u << jw;
      g = __shfl_sync(kFull, g, owner);
      if (lane == k) {
        my_e = be;
        my_g = g;
      }
    }
  }
  if (lane < K) {
    topk_idx[(size_t)t * K + lane] = my_e;
    topk_gate[(size_t)t * K + lane] = my_g;
    atomicAdd(&cnt[my_e], 1);
  }
  const unsigned ffn = __ballot_sync(kFull, lane < K && my_e < n_ffn);
  float z = 0.f;
  for (int k = 0; k < K; ++k) {
    const float gk = __shfl_sync(kFull, my_g, k);
    const int ek = __shfl_sync(kFull, my_e, k);
    if (ek >= n_ffn) z += gk;
  }
  if (lane == 0) {
    atomicAdd(&hist[__popc(ffn)], 1);
    zgate[t] = z;
  }
}

template <int J>
__device__ __forceinline__ void load_bias(const float* bias, int E, int lane,
                                          float (&bia)[J]) {
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    bia[j] = e < E ? bias[e] : 0.f;
  }
}

// WARPS tokens per CTA at a time: 8 for large batches, 1 for small ones (each token's
// dependent chain then has an SM to itself). The logits come from S split-K slices summed
// in slice order (S = 1: the logits themselves; S > 1: the sum is also written out).
template <int J, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, WARPS == 8 ? 2 : 1) k_route_topk(
    const float* src, int S, size_t slice, float* logits_out,
    const float* bias, int T, int E, int n_ffn, int K,
    int32_t* topk_idx, float* topk_gate, int32_t* counts,
    int32_t* nffn_hist, float* zgate) {
  __shared__ int s_counts[WARPS > 1 ? 1024 : 1];
  __shared__ int s_hist[33];
  __shared__ WarpScratch s_ws[WARPS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_launch_dependents();
  if constexpr (WARPS > 1) {
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_counts[i] = 0;
    if (threadIdx.x <= K) s_hist[threadIdx.x] = 0;
  }
  pdl_wait();
  __syncthreads();
  int* cnt = WARPS > 1 ? s_counts : counts;
  int* hist = WARPS > 1 ? s_hist : nffn_hist;

  float bia[J];
  load_bias<J>(bias, E, lane, bia);
  for (int t = blockIdx.x * WARPS + warp; t < T; t += gridDim.x * WARPS) {
    const float* Lr = src + (size_t)t * E;
    float lv[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      float v = -INFINITY;
      if (e < E) {
        v = Lr[e];
        for (int sp = 1; sp < S; ++sp) v += Lr[sp * slice + e];
        if (S > 1) logits_out[(size_t)t * E + e] = v;
      }
      lv[j] = v;
    }
    route_token<J>(lv, bia, lane, t, E, n_ffn, K, s_ws[warp], topk_idx, topk_gate, zgate, cnt,
                   hist);
  }
  if constexpr (WARPS > 1) {
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x)
      if (s_counts[i]) atomicAdd(&counts[i], s_counts[i]);
    if (threadIdx.x <= K && s_hist[threadIdx.x])
      atomicAdd(&nffn_hist[threadIdx.x], s_hist[threadIdx.x]);
  }
}

// Small batches with many split-K slices: one CTA per token sums the S slices of its
// logits (slice order; eight slices in flight per thread, 16-byte loads when the rows
// allow) into shared memory and writes them out; warp 0 then routes the token.
constexpr int kSumThreads = 256;

template <int W>
__device__ __forceinline__ void sum_slices(const float* row, size_t slice, int S,
                                           int n, float* out_s,
                                           float* out_g) {
  using V = typename std::conditional<W == 4, float4, float>::type;
  const V* p = reinterpret_cast<const V*>(row);
  const size_t sl = slice / W;
  for (int q = threadIdx.x; q < n; q += kSumThreads) {
    float v[W];
    {
      const V a = p[q];
      const float* f = reinterpret_cast<const float*>(&a);
#pragma unroll
      for (int i = 0; i < W; ++i) v[i] = f[i];
    }
    int sp = 1;
    for (; sp + 8 <= S; sp += 8) {
      V a[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] = p[(size_t)(sp + u) * sl + q];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float* f = reinterpret_cast<const float*>(&a[u]);
#pragma unroll
        for (int i = 0; i < W; ++i) v[i] += f[i];
      }
    }
    for (; sp < S; ++sp) {
      const V a = p[(size_t)sp * sl + q];
      const float* f = reinterpret_cast<const float*>(&a);
#pragma unroll
      for (int i = 0; i < W; ++i) v[i] += f[i];
    }
#pragma unroll
    for (int i = 0; i < W; ++i) out_s[q * W + i] = v[i];
    V o;
    float* f = reinterpret_cast<float*>(&o);
#pragma unroll
    for (int i = 0; i < W; ++i) f[i] = v[i];
    reinterpret_cast<V*>(out_g)[q] = o;
  }
}

template <int J>
__global__ void __launch_bounds__(kSumThreads, 1) k_route_topk_sum(
    const float* src, int S, size_t slice, float* logits_out,
    const float* bias, int T, int E, int n_ffn, int K,
    int32_t* topk_idx, float* topk_gate, int32_t* counts,
    int32_t* nffn_hist, float* zgate, int vec4) {
  __shared__ __align__(16) float s_l[32 * J];
  __shared__ WarpScratch s_ws;
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  if (vec4)
    sum_slices<4>(src + (size_t)t * E, slice, S, E / 4, s_l, logits_out + (size_t)t * E);
  else
    sum_slices<1>(src + (size_t)t * E, slice, S, E, s_l, logits_out + (size_t)t * E);
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  float bia[J], lv[J];
  load_bias<J>(bias, E, lane, bia);
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    lv[j] = e < E ? s_l[e] : -INFINITY;
  }
  route_token<J>(lv, bia, lane, t, E, n_ffn, K, s_ws, topk_idx, topk_gate, zgate, counts,
                 nffn_hist);
}

__global__ void k_zero2(int32_t* a, int na, int32_t* b, int nb) {
  pdl_launch_dependents();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < na; i += gridDim.x * blockDim.x) a[i] = 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x) b[i] = 0;
}

template <int J>
cudaError_t launch_topk_j(int T, int sm_count, cudaStream_t st, const float* src, int S,
                          size_t slice, float* logits_out, const float* bias, int E, int n_ffn,
                          int K, int32_t* idx, float* gate, int32_t* counts, int32_t* hist,
                          float* zgate) {
  if (T < 8 * sm_count && S > 4) {
    // 16-byte rows: E a multiple of 4 and both bases 16-byte aligned
    const int vec4 = (E % 4 == 0) && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(logits_out)) & 15) == 0;
    return launch_kernel(k_route_topk_sum<J>, T, kSumThreads, 0, st, 1, src, S, slice, logits_out,
                         bias, T, E, n_ffn, K, idx, gate, counts, hist, zgate, vec4);
  }
  if (T < 8 * sm_count)
    return launch_kernel(k_route_topk<J, 1>, T, 32, 0, st, 1, src, S, slice, logits_out, bias, T,
                         E, n_ffn, K, idx, gate, counts, hist, zgate);
  int blocks = (T + 7) / 8;
  if (blocks > 8 * sm_count) blocks = 8 * sm_count;
  return launch_kernel(k_route_topk<J, 8>, blocks, 256, 0, st, 1, src, S, slice, logits_out, bias,
                       T, E, n_ffn, K, idx, gate, counts, hist, zgate);
}
}  // namespace

bool route_topk_sums_slices(int T, int S, int sm_count) { return S <= 4 || T < 8 * sm_count; }

cudaError_t launch_zero_counts(int32_t* counts, int E, int32_t* nffn_hist, int K, cudaStream_t st) {
  const cudaError_t e = launch_kernel(k_zero2, (E + 255) / 256, 256, 0, st, 1, counts, E, nffn_hist,
                                      K + 1);
  count_launch();
  return e;
}

cudaError_t launch_route_topk(const float* src, int S, float* logits_out, const float* bias,
                              int T, int E, int n_ffn, int K, int32_t* topk_idx,
                              float* topk_gate, int32_t* counts, int32_t* nffn_hist,
                              float* zgate, int sm_count, cudaStream_t st) {
  const size_t slice = (size_t)T * E;
  const int J = (E + 31) / 32;
  cudaError_t err = cudaErrorInvalidValue;
#define MOE_TOPK_CASE(JJ)                                                                     \
  if (J <= JJ) {                                                                              \
    err = launch_topk_j<JJ>(T, sm_count, st, src, S, slice, logits_out, bias, E, n_ffn, K,    \
                            topk_idx, topk_gate, counts, nffn_hist, zgate);                   \
  } else
  MOE_TOPK_CASE(1) MOE_TOPK_CASE(2) MOE_TOPK_CASE(3) MOE_TOPK_CASE(4) MOE_TOPK_CASE(6)
  MOE_TOPK_CASE(8) MOE_TOPK_CASE(12) MOE_TOPK_CASE(16) MOE_TOPK_CASE(24) MOE_TOPK_CASE(32) {
    return cudaErrorInvalidValue;
  }
#undef MOE_TOPK_CASE
  count_launch();
  return err;
}

}  // namespace moe
