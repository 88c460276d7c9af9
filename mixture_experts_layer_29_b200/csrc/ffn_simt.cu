// ffn_simt.cu - the grouped SwiGLU FFN in fp32 on the CUDA cores, for fp32 layers (the
// tensor cores have no fp32-exact kind). Same data flow as the tensor-core path:
//   h[r, i] = silu(x_perm[r] . W_gate[e, i]) * (x_perm[r] . W_up[e, i])
//   y[r, j] = h[r] . W_down[e, j]
// then y is stored per row (deterministic combine) or s * gate * y is added atomically
// into the token's accumulator. The row count R lives on the device (offsets[n_ffn]);
// the grids cover the worst case T * K rows and rows >= R return at once.
// LongCat-Flash Technical Report digest, Key claims (report §2.4): per-expert intermediate.
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int n_ffn, int r) {
  int lo = 0, hi = n_ffn - 1;     // largest e with offsets[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(128) k_ffn_up_simt(const float* x_perm,
                                                     const int32_t* offsets,
                                                     const float* __restrict__ wgu, float* h,
                                                     int H, int I, int n_ffn) {
  pdl_launch_dependents();
  pdl_wait();
  const int R = offsets[n_ffn];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= I) return;
  for (int r = blockIdx.y; r < R; r += gridDim.y) {
    const int e = expert_of_row(offsets, n_ffn, r);
    const float* xr = x_perm + (size_t)r * H;
    const float* wg = wgu + ((size_t)e * 2 * I + i) * H;
    const float* wu = wgu + ((size_t)e * 2 * I + I + i) * H;
    float g = 0.f, u = 0.f;
    for (int k = 0; k < H; ++k) {
      const float xv = xr[k];
      g = fmaf(xv, wg[k], g);
      u = fmaf(xv, wu[k], u);
    }
    h[(size_t)r * I + i] = g / (1.0f + expf(-g)) * u;
  }
}

__global__ void __launch_bounds__(128) k_ffn_down_simt(const float* h,
                                                       const int32_t* offsets,
                                                       const float* __restrict__ wd,
                                                       const int32_t* perm_token,
                                                       const float* row_gate,
                                                       float* y_perm,
                                                       float* out_acc, int H, int I,
                                                       int n_ffn, float scale, int fused) {
  pdl_launch_dependents();
  pdl_wait();
  const int R = offsets[n_ffn];
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= H) return;
  for (int r = blockIdx.y; r < R; r += gridDim.y) {
    const int e = expert_of_row(offsets, n_ffn, r);
    const float* hr = h + (size_t)r * I;
    const float* w = wd + ((size_t)e * H + j) * I;
    float y = 0.f;
    for (int k = 0; k < I; ++k) y = fmaf(hr[k], w[k], y);
    if (fused)
      atomicAdd(out_acc + (size_t)perm_token[r] * H + j, scale * row_gate[r] * y);
    else
      y_perm[(size_t)r * H + j] = y;
  }
}

}  // namespace

cudaError_t launch_grouped_ffn_simt(const float* x_perm, const int32_t* offsets,
                                    const float* w_gate_up, const float* w_down,
                                    const int32_t* perm_token, const float* row_gate, float* h,
                                    float* y_perm, float* out_acc, int T, int H, int I,
                                    int n_ffn, int K, float scale, int fused, cudaStream_t st) {
  const int rows = T * K < 65535 ? T * K : 65535;   // rows beyond: grid-stride loop
  dim3 g1((I + 127) / 128, rows);
  cudaError_t e = launch_kernel(k_ffn_up_simt, g1, 128, 0, st, 1, x_perm, offsets, w_gate_up, h,
                                H, I, n_ffn);
  count_launch();
  if (e != cudaSuccess) return e;
  dim3 g2((H + 127) / 128, rows);
  e = launch_kernel(k_ffn_down_simt, g2, 128, 0, st, 1, h, offsets, w_down, perm_token, row_gate,
                    y_perm, out_acc, H, I, n_ffn, scale, fused);
  count_launch();
  return e;
}

}  // namespace moe
