// gemm_tc.cu - grouped bf16 GEMMs of the SwiGLU experts on the 5th-generation tensor
// cores (tcgen05.mma, TMEM accumulators, TMA-fed shared-memory ring).
//
// LongCat-Flash Technical Report digest, Key claims (report §2.4): per-expert FFN
// intermediate 2048 at hidden 6144; Method: the FFN experts of one MoE pool. The rows of
// each expert's group (from the permutation) form the A operand, the expert's weights the
// B operand; both are K-major, so one kernel shape serves
//   gate/up:  [G | U] = x_perm[rows_e] . W_gu[e]^T   then  h = silu(G) * U   (bf16)
//   down:     y = h[rows_e] . W_d[e]^T, stored per row (deterministic combine) or scaled
//             by s * gate and added atomically into the token's fp32 accumulator.
//
// Kernel structure (one CTA per SM, persistent, static round-robin over output tiles):
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 per stage (two boxes of
//               128 rows) into a 4-stage ring, 128-byte swizzle, no multicast
//   warp 1      TMEM owner and MMA issuer: 4 x tcgen05.mma M128 N256 K16 per stage,
//               tcgen05.commit frees the stage; one commit per tile hands the accumulator
//               to the epilogue
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 32 columns, math, global stores / atomics
// Two 256-column fp32 accumulators (all 512 TMEM columns) let the epilogue of one tile
// overlap the MMAs of the next.
//
// Tiles: the M tiles of expert e are ceil(count_e / 128); the tile table (prefix sum over
// experts) is built in shared memory from `offsets` by every CTA, so the host never
// reads the counts. Rows past the expert's group are computed from whatever the next
// rows hold and are never stored. Every wait is bounded; a wait that runs out writes
// MOE_ERR_TIMEOUT to the status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 48 KB
constexpr int kThreads = 192;
constexpr int kMaxExperts = 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN);

enum Mode : int { kGateUp = 0, kDownStore = 1, kDownAtomic = 2 };

struct alignas(1024) SharedStorage {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort_flag;
  int offs[kMaxExperts + 1];
  int toff[kMaxExperts + 1];
};

struct GemmArgs {
  int mode;
  int n_ffn;
  int kblocks;        // K / 64
  int n_tiles;        // N tiles per M tile
  int b_rows;         // B rows per expert: 2I (gate/up) or H (down)
  int b_second;       // row offset of the second 128-row B box: I (gate/up) or 128 (down)
  int n_valid;        // valid output columns: I (h) or H (y)
  int ld_out;         // output row length in elements
  int col_step;       // output columns per N tile: 128 (h) or 256 (y)
  const int32_t* offsets;
  void* out;
  const int32_t* perm_token;
  const float* row_gate;
  float scale;
  int* status;
};

struct Tile {
  int e, row0, row_end, nt;
};

__device__ __forceinline__ Tile decode_tile(const SharedStorage& s, const GemmArgs& g, int tile) {
  Tile t;
  const int mt = tile / g.n_tiles;
  t.nt = tile - mt * g.n_tiles;
  // largest e with toff[e] <= mt
  int lo = 0, hi = g.n_ffn - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.toff[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  t.e = lo;
  t.row0 = s.offs[lo] + (mt - s.toff[lo]) * BM;
  t.row_end = s.offs[lo + 1];
  return t;
}

__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  SharedStorage& s = *reinterpret_cast<SharedStorage*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- set-up -------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 128);
    }
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // tile table: toff[e] = sum_{e' < e} ceil(count_e' / 128)
  for (int i = threadIdx.x; i <= g.n_ffn; i += kThreads) s.offs[i] = g.offsets[i];
  __syncthreads();
  if (warp == 2) {
    const int per = (g.n_ffn + 31) / 32;
    const int b = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) local += (s.offs[b + i + 1] - s.offs[b + i] + BM - 1) / BM;
    const int inc = warp_inclusive_scan(local);
    int run = inc - local;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        s.toff[b + i] = run;
        run += (s.offs[b + i + 1] - s.offs[b + i] + BM - 1) / BM;
      }
    if (lane == 31) s.toff[g.n_ffn] = inc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = s.toff[g.n_ffn] * g.n_tiles;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0) {
    // ---- TMA producer ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const Tile t = decode_tile(s, g, tile);
        const int brow0 = t.e * g.b_rows + t.nt * (g.mode == kGateUp ? BM : BN);
        const int brow1 = brow0 + g.b_second;
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&s.full[stage], STAGE_BYTES);
          tma_load_2d(s.a[stage], &tmA, kb * BK, t.row0, &s.full[stage]);
          tma_load_2d(s.b[stage], &tmB, kb * BK, brow0, &s.full[stage]);
          tma_load_2d(s.b[stage] + B_BYTES / 2, &tmB, kb * BK, brow1, &s.full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            umma_bf16(d_tmem, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32),
                      kIdesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&s.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&s.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // ---- epilogue (warps 2..5: TMEM lane quarter = warp % 4) -----------------------------
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile t = decode_tile(s, g, tile);
      // one lane waits, the warp follows it: tcgen05.ld below needs all 32 lanes
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&s.tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      const int row = t.row0 + row_in_tile;
      const bool valid = row < t.row_end;
      if (g.mode == kGateUp) {
        __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(g.out);
#pragma unroll 1
        for (int c = 0; c < BM; c += 32) {
          uint32_t gr[32], ur[32];
          tmem_ld_32x32b_x32(tbase + c, gr);
          tmem_ld_32x32b_x32(tbase + BM + c, ur);
          tmem_ld_wait();
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hout + (size_t)row * g.ld_out + t.nt * BM + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = v * 8 + i * 2;
                const float h0 = silu_f(__uint_as_float(gr[j])) * __uint_as_float(ur[j]);
                const float h1 = silu_f(__uint_as_float(gr[j + 1])) * __uint_as_float(ur[j + 1]);
                w[i] = pack_bf16x2(h0, h1);
              }
              dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
        int tok = 0;
        float sc = 0.f;
        if (g.mode == kDownAtomic && valid) {
          tok = g.perm_token[row];
          sc = g.scale * g.row_gate[row];
        }
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t yr[32];
          tmem_ld_32x32b_x32(tbase + c, yr);
          tmem_ld_wait();
          const int col = t.nt * BN + c;
          if (valid && col < g.n_valid) {
            if (g.mode == kDownStore) {
              uint4* dst = reinterpret_cast<uint4*>(
                  static_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.ld_out + col);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int j = v * 8 + i * 2;
                  w[i] = pack_bf16x2(__uint_as_float(yr[j]), __uint_as_float(yr[j + 1]));
                }
                dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out) +
                                                      (size_t)tok * g.ld_out + col);
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                atomicAdd(dst + v, make_float4(sc * __uint_as_float(yr[4 * v + 0]),
                                               sc * __uint_as_float(yr[4 * v + 1]),
                                               sc * __uint_as_float(yr[4 * v + 2]),
                                               sc * __uint_as_float(yr[4 * v + 3])));
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s.tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- tear-down ------------------------------------------------------------------------
  if (*abort_flag) {
    set_status(g.status, MOE_ERR_TIMEOUT);
    // let copies and MMAs already in flight land before the CTA's memory goes away
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? MOE_OK : MOE_ERR_CUDA;
}

// rows x cols bf16 matrix, row-major; box = 64 columns x 128 rows, 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {BK, BM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

constexpr size_t kSmemBytes = sizeof(SharedStorage) + 1024;

int launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, int sm_count,
               cudaStream_t st) {
  if (cudaFuncSetAttribute(k_grouped_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return MOE_ERR_CUDA;
  k_grouped_gemm_tc<<<sm_count, kThreads, kSmemBytes, st>>>(ma, mb, g);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

int launch_grouped_ffn_tc(const void* x_perm, const int32_t* offsets, const void* w_gate_up,
                          const void* w_down, const int32_t* perm_token, const float* row_gate,
                          void* h, void* y_perm, float* out_acc, int T, int H, int I, int n_ffn,
                          int K, float scale, int fused, int* status, int sm_count,
                          cudaStream_t st) {
  static_assert(sizeof(SharedStorage) + 1024 <= 227 * 1024, "shared memory budget");
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  const uint64_t rows = (uint64_t)T * K + BM;   // x_perm / h / y_perm allocation rows
  CUtensorMap mx, mwgu, mh, mwd;
  int rc;
  if ((rc = make_map(&mx, x_perm, rows, H)) != MOE_OK) return rc;
  if ((rc = make_map(&mwgu, w_gate_up, (uint64_t)n_ffn * 2 * I, H)) != MOE_OK) return rc;
  if ((rc = make_map(&mh, h, rows, I)) != MOE_OK) return rc;
  if ((rc = make_map(&mwd, w_down, (uint64_t)n_ffn * H, I)) != MOE_OK) return rc;

  GemmArgs g1{};
  g1.mode = kGateUp;
  g1.n_ffn = n_ffn;
  g1.kblocks = H / BK;
  g1.n_tiles = I / BM;
  g1.b_rows = 2 * I;
  g1.b_second = I;
  g1.n_valid = I;
  g1.ld_out = I;
  g1.col_step = BM;
  g1.offsets = offsets;
  g1.out = h;
  g1.status = status;
  if ((rc = launch_one(mx, mwgu, g1, sm_count, st)) != MOE_OK) return rc;

  GemmArgs g2{};
  g2.mode = fused ? kDownAtomic : kDownStore;
  g2.n_ffn = n_ffn;
  g2.kblocks = I / BK;
  g2.n_tiles = (H + BN - 1) / BN;
  g2.b_rows = H;
  g2.b_second = BM;
  g2.n_valid = H;
  g2.ld_out = H;
  g2.col_step = BN;
  g2.offsets = offsets;
  g2.out = fused ? static_cast<void*>(out_acc) : y_perm;
  g2.perm_token = perm_token;
  g2.row_gate = row_gate;
  g2.scale = scale;
  g2.status = status;
  return launch_one(mh, mwd, g2, sm_count, st);
}

}  // namespace moe
