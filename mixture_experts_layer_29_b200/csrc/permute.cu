// permute.cu - stable permutation of the FFN picks into expert-contiguous groups.
//
// The tokens are cut into chunks of 32 (one warp). For each chunk c and FFN expert e a
// 32-bit mask holds the lanes (tokens) of the chunk that picked e. The row of pick (t, e)
// is then
//     offsets[e] + sum_{c' < c} popc(mask[e][c']) + popc(mask[e][c] & lanes_below(t)),
// which orders each group by token without any atomics that pick positions: the result
// is bit-reproducible. Kernels:
//   1. k_perm_masks    - masks [n_ffn][nchunk] (shared-memory atomicOr, order-free)
//   2. k_perm_scan     - per expert: exclusive prefix of the chunk popcounts, and counts
//   3. k_perm_scatter  - offsets (a block scan of the counts, in every CTA), perm_token,
//                        row_of, row_gate, the 16-byte vectorised copy x -> x_perm and,
//                        optionally, out_acc = zgate * x (the zero-computation experts'
//                        term: LongCat-Flash Technical Report digest, Key claims, report
//                        §2.1: a zero-computation expert is an identity map).
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kChunksPerBlock = 8;   // 8 warps x 32 tokens

// Is slot k of token t a valid, first occurrence of an expert? Writes the status word for
// an index outside [0, E) or a repeated expert; such a pick is dropped.
__device__ __forceinline__ bool valid_pick(const int32_t* idx_row, int k, int E, int* status) {
  const int e = idx_row[k];
  if (e < 0 || e >= E) {
    set_status(status, MOE_ERR_DEVICE_CHECK);
    return false;
  }
  for (int j = 0; j < k; ++j)
    if (idx_row[j] == e) {
      set_status(status, MOE_ERR_DEVICE_CHECK);
      return false;
    }
  return true;
}

__global__ void __launch_bounds__(256) k_perm_masks(const int32_t* topk_idx, int T,
                                                    int n_ffn, int E, int K, int nchunk,
                                                    uint32_t* masks, int* status) {
  extern __shared__ uint32_t sm_masks[];   // [8][n_ffn]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < kChunksPerBlock * n_ffn; i += blockDim.x) sm_masks[i] = 0u;
  pdl_wait();
  __syncthreads();
  const int c = blockIdx.x * kChunksPerBlock + warp;
  const int t = c * 32 + lane;
  if (c < nchunk && t < T) {
    const int32_t* row = topk_idx + (size_t)t * K;
    for (int k = 0; k < K; ++k) {
      if (!valid_pick(row, k, E, status)) continue;
      const int e = row[k];
      if (e < n_ffn) atomicOr(&sm_masks[warp * n_ffn + e], 1u << lane);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kChunksPerBlock * n_ffn; i += blockDim.x) {
    const int e = i / kChunksPerBlock, w = i % kChunksPerBlock;
    const int cc = blockIdx.x * kChunksPerBlock + w;
    if (cc < nchunk) masks[(size_t)e * nchunk + cc] = sm_masks[w * n_ffn + e];
  }
}

// one warp per FFN expert
__global__ void __launch_bounds__(256) k_perm_scan(const uint32_t* masks, int n_ffn,
                                                   int nchunk, int32_t* crel,
                                                   int32_t* ecount) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= n_ffn) return;
  const uint32_t* m = masks + (size_t)e * nchunk;
  int32_t* out = crel + (size_t)e * nchunk;
  int run = 0;
  for (int base = 0; base < nchunk; base += 32) {
    const int c = base + lane;
    const int v = c < nchunk ? __popc(m[c]) : 0;
    const int inc = warp_inclusive_scan(v);
    if (c < nchunk) out[c] = run + inc - v;
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) ecount[e] = run;
}

// 8 tokens per CTA (one warp each).
constexpr int kPermVec = 4;   // 16-byte vectors of x each lane loads before storing them
template <bool XBF16>
__global__ void __launch_bounds__(256) k_perm_scatter(
    const int32_t* topk_idx, const float* topk_gate,
    const float* zgate, const void* x, int T, int H, int n_ffn, int E,
    int K, int nchunk, const uint32_t* masks, const int32_t* crel,
    const int32_t* ecount, int32_t* offsets,
    int32_t* perm_token, int32_t* row_of, float* row_gate,
    void* x_perm, float* out_acc, int* status) {
  __shared__ int32_t s_off[1025];
  __shared__ int32_t s_wsum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_launch_dependents();
  pdl_wait();

  // offsets = exclusive scan of ecount[0, n_ffn): each thread owns ceil(n_ffn/256) entries
  {
    const int per = (n_ffn + 255) / 256;
    const int b = threadIdx.x * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (b + i < n_ffn) local += ecount[b + i];
    const int inc = warp_inclusive_scan(local);
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const int v = lane < 8 ? s_wsum[lane] : 0;
      const int wi = warp_inclusive_scan(v);
      if (lane < 8) s_wsum[lane] = wi - v;
    }
    __syncthreads();
    int run = s_wsum[warp] + inc - local;
    for (int i = 0; i < per; ++i)
      if (b + i < n_ffn) {
        s_off[b + i] = run;
        run += ecount[b + i];
      }
    if (threadIdx.x == 255) s_off[n_ffn] = s_wsum[7] + inc;
    __syncthreads();
    if (blockIdx.x == 0)
      for (int i = threadIdx.x; i <= n_ffn; i += blockDim.x) offsets[i] = s_off[i];
  }

  __shared__ int32_t s_rows[8][32];
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;                       // whole warp: t depends on the warp only
  const int32_t* irow = topk_idx + (size_t)t * K;
  if (lane < K) {
    int row = -1;
    const bool ok = valid_pick(irow, lane, E, nullptr);   // the masks kernel reported it
    const int e = irow[lane];
    if (ok && e < n_ffn) {
      const int c = t >> 5, l = t & 31;
      const uint32_t m = masks[(size_t)e * nchunk + c];
      row = s_off[e] + crel[(size_t)e * nchunk + c] + __popc(m & ((1u << l) - 1u));
      perm_token[row] = t;
      row_gate[row] = topk_gate[(size_t)t * K + lane];
    }
    row_of[(size_t)t * K + lane] = row;
    s_rows[warp][lane] = row;
  }
  __syncwarp();

  // copy x[t] into every FFN row of the token: each lane loads kPermVec 16-byte vectors of
  // the row (32 apart) before storing them, so that more loads are in flight per warp
  const float zg = out_acc ? zgate[t] : 0.f;
  constexpr int esz = XBF16 ? 2 : 4;
  const int nvec = H * esz / 16;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + (size_t)t * H * esz);
  if (!x_perm && !out_acc) return;
  for (int v0 = lane; v0 < nvec; v0 += 32 * kPermVec) {
    uint4 q[kPermVec];
#pragma unroll
    for (int u = 0; u < kPermVec; ++u)
      if (v0 + 32 * u < nvec) q[u] = src[v0 + 32 * u];
#pragma unroll
    for (int u = 0; u < kPermVec; ++u) {
      const int v = v0 + 32 * u;
      if (v >= nvec) break;
      if (x_perm) {
        for (int k = 0; k < K; ++k) {
          const int r = s_rows[warp][k];
          if (r >= 0)
            reinterpret_cast<uint4*>(static_cast<char*>(x_perm) + (size_t)r * H * esz)[v] = q[u];
        }
      }
      if (out_acc) {
        float* o = out_acc + (size_t)t * H + (size_t)v * (16 / esz);
        if (XBF16) {
          const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&q[u]);
          reinterpret_cast<float4*>(o)[0] = make_float4(zg * to_f32(b[0]), zg * to_f32(b[1]),
                                                        zg * to_f32(b[2]), zg * to_f32(b[3]));
          reinterpret_cast<float4*>(o)[1] = make_float4(zg * to_f32(b[4]), zg * to_f32(b[5]),
                                                        zg * to_f32(b[6]), zg * to_f32(b[7]));
        } else {
          const float* f = reinterpret_cast<const float*>(&q[u]);
          reinterpret_cast<float4*>(o)[0] = make_float4(zg * f[0], zg * f[1], zg * f[2], zg * f[3]);
        }
      }
    }
  }
}

// ---- small batches (T <= 512): all index work in one CTA, then a wide copy kernel -------
constexpr int kSmallT = 512;

// One CTA of 512 threads: bitmasks [n_ffn][16] and their per-expert prefixes in shared
// memory, the expert counts, the offsets (block scan), then every pick's row. The same
// ranking as the three-kernel path, so the same rows.
__global__ void __launch_bounds__(512) k_perm_index_small(
    const int32_t* topk_idx, const float* topk_gate, int T, int n_ffn,
    int E, int K, int32_t* offsets, int32_t* perm_token,
    int32_t* row_of, float* row_gate, int* status) {
  extern __shared__ uint32_t sm[];
  const int nch = (T + 31) / 32;                                 // 32-token chunks (<= 16)
  uint32_t* masks = sm;                                          // [n_ffn][nch]
  int32_t* crel = reinterpret_cast<int32_t*>(sm + n_ffn * nch);  // [n_ffn][nch]
  int32_t* offs = crel + n_ffn * nch;                            // [n_ffn + 1]
  __shared__ int32_t s_wsum[16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  for (int i = tid; i < n_ffn * nch; i += blockDim.x) masks[i] = 0u;
  pdl_wait();
  __syncthreads();
  const int t = tid;          // warp w holds the tokens of chunk w, lane = token bit
  // keep[k]: slot k is in range and the first slot of its expert (a repeated expert shows
  // as its bit already set: a token's own slots run in order, other tokens use other bits)
  uint32_t keep = 0u;
  int ek[32];
  if (t < T) {
    const int32_t* row = topk_idx + (size_t)t * K;
#pragma unroll
    for (int k = 0; k < 32; ++k) ek[k] = k < K ? row[k] : -1;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if (k >= K) break;
      const int e = ek[k];
      if (e < 0 || e >= E) {
        set_status(status, MOE_ERR_DEVICE_CHECK);
        continue;
      }
      if (e < n_ffn) {
        const uint32_t bit = 1u << lane;
        if (atomicOr(&masks[e * nch + warp], bit) & bit) {
          set_status(status, MOE_ERR_DEVICE_CHECK);
          continue;
        }
      } else {
        // zero experts have no mask: repeated zero experts are checked directly
        bool dup = false;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < k && ek[j] == e) dup = true;
        if (dup) {
          set_status(status, MOE_ERR_DEVICE_CHECK);
          continue;
        }
      }
      keep |= 1u << k;
    }
  }
  __syncthreads();
  // per expert: exclusive prefix of the chunk popcounts, and the count
  int local = 0;
  for (int e = tid; e < n_ffn; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < nch; ++c) {
      crel[e * nch + c] = run;
      run += __popc(masks[e * nch + c]);
    }
    offs[e] = run;          // count for now
  }
  __syncthreads();
  // offsets: exclusive scan of the counts (each thread a contiguous run of experts)
  const int per = (n_ffn + blockDim.x - 1) / blockDim.x;
  const int b = tid * per;
  for (int i = 0; i < per; ++i)
    if (b + i < n_ffn) local += offs[b + i];
  const int inc = warp_inclusive_scan(local);
  if (lane == 31) s_wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < 16 ? s_wsum[lane] : 0;
    const int wi = warp_inclusive_scan(v);
    if (lane < 16) s_wsum[lane] = wi - v;
  }
  __syncthreads();
  int run = s_wsum[warp] + inc - local;
  int cnt[4];
  for (int i = 0; i < per && i < 4; ++i) cnt[i] = (b + i < n_ffn) ? offs[b + i] : 0;
  __syncthreads();
  for (int i = 0; i < per && i < 4; ++i)
    if (b + i < n_ffn) {
      offs[b + i] = run;
      run += cnt[i];
    }
  if (tid == blockDim.x - 1) offs[n_ffn] = run;
  __syncthreads();
  for (int i = tid; i <= n_ffn; i += blockDim.x) offsets[i] = offs[i];
  if (t < T) {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      if (k >= K) break;
      int r = -1;
      const int e = ek[k];
      if (((keep >> k) & 1u) && e < n_ffn) {
        const int c = t >> 5;
        r = offs[e] + crel[e * nch + c] +
            __popc(masks[e * nch + c] & ((1u << (t & 31)) - 1u));
        perm_token[r] = t;
        row_gate[r] = topk_gate[(size_t)t * K + k];
      }
      row_of[(size_t)t * K + k] = r;
    }
  }
}

// Copy x[t] into the rows of its FFN picks (and out_acc = zgate * x): block (t, seg) takes
// one contiguous slice of the row, 16 bytes per thread per step.
template <bool XBF16>
__global__ void __launch_bounds__(128) k_perm_copy(const int32_t* row_of,
                                                   const float* zgate,
                                                   const void* x, int H, int K,
                                                   void* x_perm,
                                                   float* out_acc) {
  __shared__ int32_t s_rows[32];
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  if (threadIdx.x < K) s_rows[threadIdx.x] = row_of[(size_t)t * K + threadIdx.x];
  __syncthreads();
  constexpr int esz = XBF16 ? 2 : 4;
  const int nvec = H * esz / 16;
  const int per = (nvec + gridDim.y - 1) / gridDim.y;
  const int v_end = min(nvec, (int)(blockIdx.y + 1) * per);
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + (size_t)t * H * esz);
  const float zg = out_acc ? zgate[t] : 0.f;
  for (int v = blockIdx.y * per + threadIdx.x; v < v_end; v += blockDim.x) {
    const uint4 q = src[v];
    if (x_perm)
      for (int k = 0; k < K; ++k) {
        const int r = s_rows[k];
        if (r >= 0) reinterpret_cast<uint4*>(static_cast<char*>(x_perm) + (size_t)r * H * esz)[v] = q;
      }
    if (out_acc) {
      float* o = out_acc + (size_t)t * H + (size_t)v * (16 / esz);
      if (XBF16) {
        const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&q);
        reinterpret_cast<float4*>(o)[0] =
            make_float4(zg * to_f32(b[0]), zg * to_f32(b[1]), zg * to_f32(b[2]), zg * to_f32(b[3]));
        reinterpret_cast<float4*>(o)[1] =
            make_float4(zg * to_f32(b[4]), zg * to_f32(b[5]), zg * to_f32(b[6]), zg * to_f32(b[7]));
      } else {
        const float* f = reinterpret_cast<const float*>(&q);
        reinterpret_cast<float4*>(o)[0] = make_float4(zg * f[0], zg * f[1], zg * f[2], zg * f[3]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute(const int32_t* topk_idx, const float* topk_gate, const float* zgate,
                           const void* x, int x_is_bf16, int T, int H, int n_ffn, int E, int K,
                           uint32_t* masks, int32_t* crel, int32_t* ecount, int32_t* offsets,
                           int32_t* perm_token, int32_t* row_of, float* row_gate, void* x_perm,
                           float* out_acc, int* status, cudaStream_t st) {
  if (T <= kSmallT && n_ffn <= 1024) {
    // one CTA for the indices, then a wide copy (short chain for small batches)
    const size_t smem = sizeof(uint32_t) * (size_t)n_ffn * ((T + 31) / 32) * 2 + sizeof(int32_t) * (n_ffn + 1);
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(k_perm_index_small,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_kernel(k_perm_index_small, 1, 512, smem, st, 1, topk_idx, topk_gate, T,
                                  n_ffn, E, K, offsets, perm_token, row_of, row_gate, status);
    count_launch();
    if (e != cudaSuccess) return e;
    if (x_perm || out_acc) {
      const int nvec = H * (x_is_bf16 ? 2 : 4) / 16;
      int nseg = (4 * 148 + T - 1) / T;                 // about four CTAs per SM in total
      const int max_seg = (nvec + 127) / 128;
      if (nseg > max_seg) nseg = max_seg;
      if (nseg < 1) nseg = 1;
      const dim3 grid(T, nseg);
      e = launch_kernel(x_is_bf16 ? k_perm_copy<true> : k_perm_copy<false>, grid, 128, 0, st, 1,
                        row_of, zgate, x, H, K, x_perm, out_acc);
      count_launch();
    }
    return e;
  }
  const int nchunk = (T + 31) / 32;
  const int g1 = (nchunk + kChunksPerBlock - 1) / kChunksPerBlock;
  const size_t sm1 = sizeof(uint32_t) * kChunksPerBlock * n_ffn;
  if (sm1 > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_perm_masks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_kernel(k_perm_masks, g1, 256, sm1, st, 1, topk_idx, T, n_ffn, E, K,
                                nchunk, masks, status);
  count_launch();
  if (e != cudaSuccess) return e;
  e = launch_kernel(k_perm_scan, (n_ffn + 7) / 8, 256, 0, st, 1, masks, n_ffn, nchunk, crel,
                    ecount);
  count_launch();
  if (e != cudaSuccess) return e;
  const int g3 = (T + 7) / 8;
  e = launch_kernel(x_is_bf16 ? k_perm_scatter<true> : k_perm_scatter<false>, g3, 256, 0, st, 1,
                    topk_idx, topk_gate, zgate, x, T, H, n_ffn, E, K, nchunk, masks, crel, ecount,
                    offsets, perm_token, row_of, row_gate, x_perm, out_acc, status);
  count_launch();
  return e;
}

}  // namespace moe
