// gemm_bwd.cu - the expert GEMMs of the layer's backward on the 5th-generation tensor cores.
//
// With dy[r] = s * g * dout[token of r] on every FFN row r of expert e (see backward.cu):
//   kDH  dh = dy . W_d[e]          M = rows of e, K = H, N = I; B = W_d[e] read N-major,
//        then the SwiGLU backward in the epilogue from the recomputed G, U of the row:
//        dG = dh * U * sig(G) * (1 + G (1 - sig(G))),  dU = dh * G * sig(G)  -> dgu [dG | dU]
//   kDX  dx_perm = dgu . W_gu[e]   M = rows of e, K = 2I, N = H; B = W_gu[e] N-major; fp32
//   kDW  d_down[e]    = dy_e^T  h_e       M = H,  K = rows of e, N = I
//        d_gate_up[e] = dgu_e^T x_perm_e  M = 2I, K = rows of e, N = H
//        A and B both MN-major (the row buffers read along their rows); fp32, written for
//        the experts that have rows only. The experts' kDW runs on CTA pairs
//        (k_bwd_wgrad_pair, 256 x 256 tiles); k_bwd_gemm keeps the router's and serves
//        when MOE_TUNE_BWD_PAIR is 0 or 2.
// The forward's SwiGLU expert (LongCat-Flash Technical Report digest, Key claims, report
// §2.4: per-expert intermediate 2048 at hidden 6144) differentiated with the selection held
// fixed.
//
// Same structure as the forward kernel (one CTA per SM, persistent, warp 0 TMA producer,
// warp 1 TMEM owner + single-thread tcgen05.mma issuer, warps 2-9 epilogue, 4-stage ring
// of 48 KB, two 256-column fp32 accumulators, every wait bounded). MN-major operands come
// in as 64 K-rows x 64 MN-elements TMA boxes with the 128-byte swizzle, stacked along MN
// 8 KB apart; the shared-memory descriptor then has leading byte offset 8 KB (between MN
// blocks) and stride byte offset 1 KB (between 8-row K groups), and the instruction
// descriptor marks the operand MN-major. kDW's K runs over one expert's rows: the last
// k-block of an expert holds rows of the next one, so its tiles land on a side barrier,
// the producer warp zeroes the K-rows past the expert in shared memory, fences them to the
// async proxy and only then releases the stage to the MMA.
#include <cuda.h>

#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BOX_BYTES = 64 * BK * 2;               // one 64 x 64 box: 8 KB
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kFixWarp = 2 + kEpiWarps;             // zeroes an expert's tail K-rows
constexpr int kThreads = 64 + kEpiThreads + 32;
constexpr int kMaxExperts = 1024;
constexpr uint32_t kTmemCols = 512;

enum BwdMode : int { kDH = 0, kDX = 1, kDW = 2 };

struct BwdArgs {
  int mode;
  int n_ffn;
  int kblocks;            // kDH / kDX: K / 64
  int m_tiles;            // kDW: M / 128 (256 on CTA pairs), rounded up
  int n_tiles;            // N / 256 (rounded up)
  int b_krows;            // kDH / kDX: K rows of B per expert in its 2-D view
  int n_valid;            // output columns N
  long long ld_out;       // output row length (elements)
  long long out_expert;   // kDW: elements per expert of the output
  int I;                  // kDH: G at column c, U at column I + c of gu and dgu
  int m_valid;            // kDW: output rows M
  int b_kwrap;            // kDW: B's row is the K row modulo this (0: no wrap)
  int m_group;            // kDW: 0, or M tiles per group (N tiles outer within a group)
  int mix_rows;           // pair kDW: 0, or experts of at most this many rows take every
                          // other tile (see decode_w)
  const int32_t* offsets;
  const __nv_bfloat16* gu;
  void* out;
  int* status;
};

struct Tile {
  int e, row0, row_end, mt, nt;
};

struct alignas(1024) Smem {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t landed[STAGES];      // kDW last k-block: TMA bytes land here first
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort_flag;
  int offs[kMaxExperts + 1];
  int toff[kMaxExperts + 1];    // kDH / kDX: prefix of ceil(count / 128); kDW: of (count > 0)
  alignas(16) float stg[kEpiWarps][32][16];   // read and written as float4
};
static_assert(offsetof(Smem, stg) % 16 == 0, "staging rows are accessed as float4");

template <class S>
__device__ __forceinline__ Tile decode(const S& s, const BwdArgs& g, int tile) {
  Tile t;
  int unit;
  if (g.mode == kDW) {
    const int per = g.m_tiles * g.n_tiles;
    unit = tile / per;
    const int rem = tile - unit * per;
    if (g.m_group > 0) {
      // groups of m_group M tiles (the last one may be short); within a group the M tile
      // runs fastest, so a wave of consecutive tiles spans fewer B columns
      const int grp = rem / (g.m_group * g.n_tiles);
      const int m0 = grp * g.m_group;
      const int gsz = min(g.m_group, g.m_tiles - m0);
      const int r2 = rem - grp * g.m_group * g.n_tiles;
      t.nt = r2 / gsz;
      t.mt = m0 + (r2 - t.nt * gsz);
    } else {
      t.mt = rem / g.n_tiles;
      t.nt = rem - t.mt * g.n_tiles;
    }
  } else {
    unit = tile / g.n_tiles;
    t.nt = tile - unit * g.n_tiles;
    t.mt = 0;
  }
  // largest e with toff[e] <= unit (experts without tiles share the next one's toff)
  int lo = 0, hi = g.n_ffn - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.toff[mid] <= unit) lo = mid; else hi = mid - 1;
  }
  t.e = lo;
  t.row0 = g.mode == kDW ? s.offs[lo] : s.offs[lo] + (unit - s.toff[lo]) * BM;
  t.row_end = s.offs[lo + 1];
  return t;
}

__device__ __forceinline__ int kblocks_of(const BwdArgs& g, const Tile& t) {
  return g.mode == kDW ? (t.row_end - t.row0 + BK - 1) / BK : g.kblocks;
}

// kDW: K-rows of k-block kb that belong to the tile's expert (64 for the other modes). The
// MMA runs ceil(valid / 16) K = 16 steps; the rows in [valid, ceil16(valid)) hold the next
// expert's data and are zeroed in shared memory first (a "fix" block).
__device__ __forceinline__ int kvalid(const BwdArgs& g, const Tile& t, int kb) {
  return g.mode == kDW ? min(BK, t.row_end - (t.row0 + kb * BK)) : BK;
}
__device__ __forceinline__ bool fix_block(int valid) { return (valid & 15) != 0; }

// fp32 row stores through the warp's staging block: this thread's row holds 16 values at
// output columns [col, col + 16); a warp store then covers 8 rows x 64 bytes. A staging row
// is 16 floats, and its 16-byte chunk ch sits at chunk ch ^ ((row >> 1) & 3): each group of 8
// lanes then touches 32 distinct banks, both when a lane writes its row and when 8 lanes
// read two rows.
__device__ __forceinline__ int stg_chunk(int row, int ch) { return 4 * (ch ^ ((row >> 1) & 3)); }

__device__ __forceinline__ void store_f32_16(float (*stg)[16], int lane, const float* v,
                                             float* out, long long ld, int row_base,
                                             int row_end, int col, int n_valid) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(&stg[lane][stg_chunk(lane, i)]) =
        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * i + (lane >> 2), c = col + 4 * (lane & 3);
    const int grow = row_base + r;
    if (grow < row_end && c < n_valid)
      *reinterpret_cast<float4*>(out + (size_t)grow * ld + c) =
          *reinterpret_cast<const float4*>(&stg[r][stg_chunk(r, lane & 3)]);
  }
  __syncwarp();
}

// fp32 stores of 32 columns [col, col + 32) of this warp's 32 rows (this thread's row holds
// them in v) as full 128-byte lines: two passes of 16 rows through a 16 x 32 staging block,
// whose 16-byte chunk c of row r sits at chunk c ^ (r & 7). The lanes of a pass write their
// rows, then each warp store covers 4 rows x 128 bytes.
__device__ __forceinline__ void store_f32_32(float (*stg)[32], int lane, const uint32_t* v,
                                             float* out, long long ld, int row_base,
                                             int row_end, int col, int n_valid) {
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    if ((lane >> 4) == p) {
      const int r = lane & 15;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(&stg[r][4 * (c ^ (r & 7))]) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * i + (lane >> 3), ch = lane & 7;
      const int grow = row_base + 16 * p + r, c = col + 4 * ch;
      if (grow < row_end && c < n_valid)
        *reinterpret_cast<float4*>(out + (size_t)grow * ld + c) =
            *reinterpret_cast<const float4*>(&stg[r][4 * (ch ^ (r & 7))]);
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_bwd_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const BwdArgs g) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.landed[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], kEpiThreads);
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
  pdl_wait();
  for (int i = threadIdx.x; i <= g.n_ffn; i += kThreads) s.offs[i] = g.offsets[i];
  __syncthreads();
  if (warp == 2) {
    const int per = (g.n_ffn + 31) / 32;
    const int b = lane * per;
    auto units = [&](int e) {
      const int c = s.offs[e + 1] - s.offs[e];
      return g.mode == kDW ? (c > 0 ? 1 : 0) : (c + BM - 1) / BM;
    };
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) local += units(b + i);
    const int inc = warp_inclusive_scan(local);
    int run = inc - local;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        s.toff[b + i] = run;
        run += units(b + i);
      }
    if (lane == 31) s.toff[g.n_ffn] = inc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles =
      s.toff[g.n_ffn] * (g.mode == kDW ? g.m_tiles * g.n_tiles : g.n_tiles);
  volatile int* abort_flag = &s.abort_flag;
  const bool a_mn = g.mode == kDW;

  if (warp == 0) {
    // ---- TMA producer (lane 0) -----------------------------------------------------------
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles && !*abort_flag; tile += gridDim.x) {
      const Tile t = decode(s, g, tile);
      const int nkb = kblocks_of(g, t);
      for (int kb = 0; kb < nkb; ++kb) {
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        // a fix block lands on the side barrier; the fix warp releases it to the MMA
        uint64_t* bar = fix_block(kvalid(g, t, kb)) ? &s.landed[stage] : &s.full[stage];
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, STAGE_BYTES);
          if (a_mn) {
            const int y = t.row0 + kb * BK;
            const int yb = g.b_kwrap > 0 ? y % g.b_kwrap : y;
            tma_load_2d(s.a[stage], &tmA, t.mt * BM, y, bar);
            tma_load_2d(s.a[stage] + BOX_BYTES, &tmA, t.mt * BM + 64, y, bar);
            for (int j = 0; j < 4; ++j)
              tma_load_2d(s.b[stage] + j * BOX_BYTES, &tmB, t.nt * BN + 64 * j, yb, bar);
          } else {
            tma_load_2d(s.a[stage], &tmA, kb * BK, t.row0, bar);
            const int y = t.e * g.b_krows + kb * BK;
            for (int j = 0; j < 4; ++j)
              tma_load_2d(s.b[stage] + j * BOX_BYTES, &tmB, t.nt * BN + 64 * j, y, bar);
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer -----------------------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_major(BM, BN, a_mn, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const Tile t = decode(s, g, tile);
        const int nkb = kblocks_of(g, t);
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          const int nk = (kvalid(g, t, kb) + 15) / 16;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            if (k >= nk) break;
            const uint64_t ad = a_mn ? sw128_mnmajor_desc(a0 + k * 2048, BOX_BYTES)
                                     : sw128_kmajor_desc(a0 + k * 32);
            umma_bf16(d_tmem, ad, sw128_mnmajor_desc(b0 + k * 2048, BOX_BYTES), idesc,
                      (kb > 0 || k > 0) ? 1u : 0u);
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
  } else if (warp == kFixWarp) {
    // ---- fix warp: follows the producer's k-blocks; on each fix block it waits for the
    // TMA bytes, zeroes K-rows [valid, ceil16(valid)) of the six boxes, fences them to the
    // async proxy and releases the stage to the MMA
    if (a_mn) {
      int stage = 0;
      uint32_t landed_phase = 0;   // bit i: parity of the next completion of landed[i]
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const Tile t = decode(s, g, tile);
        const int nkb = kblocks_of(g, t);
        for (int kb = 0; kb < nkb; ++kb) {
          const int valid = kvalid(g, t, kb);
          if (fix_block(valid)) {
            int w_ok = 1;
            if (lane == 0)
              w_ok = mbar_wait(&s.landed[stage], (landed_phase >> stage) & 1u, abort_flag) ? 1 : 0;
            landed_phase ^= 1u << stage;
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
              ok = false;
              break;
            }
            const int nrow = ((valid + 15) & ~15) - valid;
            for (int i = lane; i < 6 * nrow * 8; i += 32) {
              const int box = i / (nrow * 8), rem = i - box * nrow * 8;
              const int r = valid + rem / 8, c16 = rem & 7;
              uint8_t* base = box < 2 ? s.a[stage] + box * BOX_BYTES : s.b[stage] + (box - 2) * BOX_BYTES;
              *reinterpret_cast<uint4*>(base + r * 128 + c16 * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.full[stage]);
          }
          if (++stage == STAGES) stage = 0;
        }
      }
    }
  } else {
    // ---- epilogue: TMEM lane quarter q = warp % 4, column half h = (warp - 2) / 4 ---------
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    float (*stg)[16] = s.stg[warp - 2];
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile t = decode(s, g, tile);
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(&s.tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      // kDH / kDX: output row = the tile's row; kDW: the weight row mt * 128 + q * 32 + lane
      const int row_base = g.mode == kDW ? t.mt * BM + q * 32 : t.row0 + q * 32;
      const int row_end = g.mode == kDW ? g.m_valid : t.row_end;
      const int row = row_base + lane;
#pragma unroll 1
      for (int c = 128 * h; c < 128 * h + 128; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c, v);
        tmem_ld_wait();
        const int col = t.nt * BN + c;
        if (g.mode == kDH) {
          if (row < row_end && col < g.n_valid) {
            const __nv_bfloat16* gr = g.gu + (size_t)row * 2 * g.I + col;
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.out) + (size_t)row * 2 * g.I + col;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              const uint4 G4 = *reinterpret_cast<const uint4*>(gr + 8 * q8);
              const uint4 U4 = *reinterpret_cast<const uint4*>(gr + g.I + 8 * q8);
              const __nv_bfloat16* Gb = reinterpret_cast<const __nv_bfloat16*>(&G4);
              const __nv_bfloat16* Ub = reinterpret_cast<const __nv_bfloat16*>(&U4);
              float dG[8], dU[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                swiglu_backward(__bfloat162float(Gb[i]), __bfloat162float(Ub[i]),
                                __uint_as_float(v[8 * q8 + i]), dG[i], dU[i]);
              }
              *reinterpret_cast<uint4*>(dst + 8 * q8) =
                  make_uint4(pack_bf16x2(dG[0], dG[1]), pack_bf16x2(dG[2], dG[3]),
                             pack_bf16x2(dG[4], dG[5]), pack_bf16x2(dG[6], dG[7]));
              *reinterpret_cast<uint4*>(dst + g.I + 8 * q8) =
                  make_uint4(pack_bf16x2(dU[0], dU[1]), pack_bf16x2(dU[2], dU[3]),
                             pack_bf16x2(dU[4], dU[5]), pack_bf16x2(dU[6], dU[7]));
            }
          }
        } else {
          float* out = static_cast<float*>(g.out) +
                       (g.mode == kDW ? (size_t)t.e * g.out_expert : (size_t)0);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          store_f32_16(stg, lane, f, out, g.ld_out, row_base, row_end, col, g.n_valid);
          store_f32_16(stg, lane, f + 16, out, g.ld_out, row_base, row_end, col + 16, g.n_valid);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  if (*abort_flag) {
    set_status(g.status, MOE_ERR_TIMEOUT);
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

int launch(const CUtensorMap& ma, const CUtensorMap& mb, const BwdArgs& g, int sm_count,
           cudaStream_t st) {
  constexpr size_t smem = sizeof(Smem) + 1024;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  if (cudaFuncSetAttribute(k_bwd_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  const cudaError_t e = launch_kernel(k_bwd_gemm, sm_count, kThreads, smem, st, 1, ma, mb, g);
  count_launch();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---- weight gradients on CTA pairs ----------------------------------------------------------
// d_down[e] = dy_e^T h_e and d_gate_up[e] = dgu_e^T x_perm_e as 256 x 256 tiles on a cluster
// of two CTAs (tcgen05 cta_group::2). CTA r loads the weight rows [256 mt + 128 r, +128) of
// A and the columns [256 nt + 128 r, +128) of B, both MN-major (two 64 x 64 boxes each, 8 KB
// apart), and keeps its 128 rows of the fp32 accumulator in its own TMEM; the leader issues
// the MMAs. Per SM and k-block that is 32 KB of operands against the one-CTA tile's 48 KB.
// The last k-block of an expert whose row count is not a multiple of 16: each CTA lands its
// four boxes on a barrier of its own, zeroes the K-rows past the expert and fences them to
// the async proxy. The peer's fix warp then arrives on the leader's `pfix` barrier (release
// at cluster scope); the leader's fix warp acquires it and releases the stage to the MMA.
constexpr int WBM = 256;                               // weight rows of a pair tile

// K rows per stage WK (64 or 128; MOE_TUNE_BWD_WGRAD_BK): each operand half of a CTA is two
// boxes of WK K-rows x 64 MN elements (the 128-byte swizzle caps an MN-major box at 64
// elements), so a stage holds 32 KB (WK = 64, six stages) or 64 KB (WK = 128, three).
template <int WK>
struct WCfg {
  static constexpr int STAGES = 6 * 64 / WK;
  static constexpr int BOX = WK * 128;                 // one box: WK rows of 128 bytes
  static constexpr int HALF = 2 * BOX;                 // 128 MN elements
};

template <int WK>
struct alignas(1024) WSmem {
  static constexpr int STAGES = WCfg<WK>::STAGES;
  uint8_t a[STAGES][WCfg<WK>::HALF];
  uint8_t b[STAGES][WCfg<WK>::HALF];
  uint64_t full[STAGES];        // leader: both CTAs' TMA bytes, or its fix warp on fix blocks
  uint64_t empty[STAGES];       // the leader's MMA commit, in both CTAs
  uint64_t landed[STAGES];      // fix blocks: this CTA's TMA bytes
  uint64_t pfix[STAGES];        // leader: the peer's fix warp is done with the stage
  uint64_t tfull[2];
  uint64_t tempty[2];           // leader: both CTAs' epilogue warps
  uint32_t tmem_base;
  int abort_flag;
  int n_heavy, n_light;         // experts with rows, more / at most mix_rows of them
  int offs[kMaxExperts + 1];
  int16_t order[kMaxExperts];   // the heavy experts, then the light ones, each by index
  alignas(16) float stg[kEpiWarps][16][32];   // read and written as float4
};
static_assert(offsetof(WSmem<64>, stg) % 16 == 0 && offsetof(WSmem<128>, stg) % 16 == 0,
              "staging rows are accessed as float4");
static_assert(offsetof(WSmem<64>, b) % 1024 == 0 && offsetof(WSmem<128>, b) % 1024 == 0 &&
                  WCfg<64>::HALF % 1024 == 0, "128-byte swizzled boxes need 1024-byte alignment");

// k-blocks of WK rows of a tile's expert, and the rows of k-block kb that belong to it
template <int WK>
__device__ __forceinline__ int w_kblocks(const Tile& t) { return (t.row_end - t.row0 + WK - 1) / WK; }
template <int WK>
__device__ __forceinline__ int w_kvalid(const Tile& t, int kb) {
  return min(WK, t.row_end - (t.row0 + kb * WK));
}

// Tile `tile` of the pair kernel: per expert m_tiles x n_tiles tiles. With light experts
// (mix_rows), tiles alternate between the heavy and the light ones while both last, so
// that the store-bound tiles of experts with few rows run beside MMA-bound ones; then the
// rest of the longer list.
template <class S>
__device__ __forceinline__ Tile decode_w(const S& s, const BwdArgs& g, int tile) {
  const int per = g.m_tiles * g.n_tiles;
  const int nh = s.n_heavy * per, nl = s.n_light * per;
  const int m = min(nh, nl);
  int j;
  bool light;
  if (tile < 2 * m) {
    light = (tile & 1) != 0;
    j = tile >> 1;
  } else {
    light = nl > nh;
    j = tile - m;
  }
  const int unit = j / per;
  const int rem = j - unit * per;
  Tile t;
  t.e = s.order[(light ? s.n_heavy : 0) + unit];
  t.row0 = s.offs[t.e];
  t.row_end = s.offs[t.e + 1];
  if (g.m_group > 0) {
    const int grp = rem / (g.m_group * g.n_tiles);
    const int m0 = grp * g.m_group;
    const int gsz = min(g.m_group, g.m_tiles - m0);
    const int r2 = rem - grp * g.m_group * g.n_tiles;
    t.nt = r2 / gsz;
    t.mt = m0 + (r2 - t.nt * gsz);
  } else {
    t.mt = rem / g.n_tiles;
    t.nt = rem - t.mt * g.n_tiles;
  }
  return t;
}

template <int WK>
__global__ void __launch_bounds__(kThreads, 1)
    k_bwd_wgrad_pair(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const BwdArgs g) {
  constexpr int STAGES = WCfg<WK>::STAGES, WBOX = WCfg<WK>::BOX, WHALF = WCfg<WK>::HALF;
  extern __shared__ uint8_t smem_raw[];
  WSmem<WK>& s = *reinterpret_cast<WSmem<WK>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();            // 0: leader, 1: peer
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.landed[i], 1);
      mbar_init(&s.pfix[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 2 * kEpiWarps);
    }
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  pdl_wait();
  for (int i = threadIdx.x; i <= g.n_ffn; i += kThreads) s.offs[i] = g.offsets[i];
  __syncthreads();
  cluster_sync();                                     // both CTAs' barriers initialised
  if (warp == 1) {
    tmem_alloc_pair(&s.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 2) {
    // the experts with rows, heavy ones first, each list in index order; lane l takes a
    // contiguous run of experts
    const int per = (g.n_ffn + 31) / 32;
    const int b = lane * per;
    auto cls = [&](int e) {     // 0: no rows, 1: heavy, 2: light
      const int c = s.offs[e + 1] - s.offs[e];
      return c <= 0 ? 0 : (g.mix_rows > 0 && c <= g.mix_rows ? 2 : 1);
    };
    int nh = 0, nl = 0;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        const int c = cls(b + i);
        nh += c == 1 ? 1 : 0;
        nl += c == 2 ? 1 : 0;
      }
    const int hinc = warp_inclusive_scan(nh);
    const int linc = warp_inclusive_scan(nl);
    const int h_all = __shfl_sync(0xffffffffu, hinc, 31);
    int hrun = hinc - nh, lrun = h_all + linc - nl;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        const int c = cls(b + i);
        if (c == 1) s.order[hrun++] = static_cast<int16_t>(b + i);
        else if (c == 2) s.order[lrun++] = static_cast<int16_t>(b + i);
      }
    if (lane == 31) {
      s.n_heavy = hinc;
      s.n_light = linc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = (s.n_heavy + s.n_light) * g.m_tiles * g.n_tiles;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0) {
    // ---- TMA producer (both CTAs): this CTA's weight rows of A and its columns of B ------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total_tiles && !*abort_flag; tile += nclusters) {
        const Tile t = decode_w(s, g, tile);
        const int nkb = w_kblocks<WK>(t);
        const int ax = t.mt * WBM + static_cast<int>(rank) * 128;
        const int bx = t.nt * BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int y = t.row0 + kb * WK;
          if (fix_block(w_kvalid<WK>(t, kb))) {
            uint64_t* bar = &s.landed[stage];
            mbar_arrive_expect_tx(bar, 2 * WHALF);
            tma_load_2d(s.a[stage], &tmA, ax, y, bar);
            tma_load_2d(s.a[stage] + WBOX, &tmA, ax + 64, y, bar);
            tma_load_2d(s.b[stage], &tmB, bx, y, bar);
            tma_load_2d(s.b[stage] + WBOX, &tmB, bx + 64, y, bar);
          } else {
            // the leader expects both CTAs' bytes
            const uint32_t full_leader = mapa_shared(smem_u32(&s.full[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], 4 * WHALF);
            tma_load_2d_pair(s.a[stage], &tmA, ax, y, full_leader);
            tma_load_2d_pair(s.a[stage] + WBOX, &tmA, ax + 64, y, full_leader);
            tma_load_2d_pair(s.b[stage], &tmB, bx, y, full_leader);
            tma_load_2d_pair(s.b[stage] + WBOX, &tmB, bx + 64, y, full_leader);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (leader only) ---------------------------------------------------------
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_major(WBM, BN, true, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total_tiles && !*abort_flag; tile += nclusters) {
        const Tile t = decode_w(s, g, tile);
        const int nkb = w_kblocks<WK>(t);
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          const int nk = (w_kvalid<WK>(t, kb) + 15) / 16;
#pragma unroll
          for (int k = 0; k < WK / 16; ++k) {
            if (k >= nk) break;
            umma_bf16_pair(d_tmem, sw128_mnmajor_desc(a0 + k * 2048, WBOX),
                           sw128_mnmajor_desc(b0 + k * 2048, WBOX), idesc,
                           (kb > 0 || k > 0) ? 1u : 0u);
          }
          const uint32_t e_local = smem_u32(&s.empty[stage]);
          umma_commit_pair(mapa_shared(e_local, 0));
          umma_commit_pair(mapa_shared(e_local, 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        const uint32_t f_local = smem_u32(&s.tfull[acc]);
        umma_commit_pair(mapa_shared(f_local, 0));
        umma_commit_pair(mapa_shared(f_local, 1));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else if (warp == kFixWarp) {
    // ---- fix warp (both CTAs): zeroes the K-rows past the expert on fix blocks ------------
    int stage = 0;
    uint32_t landed_phase = 0;   // bit i: parity of the next completion of landed[i]
    uint32_t pfix_phase = 0;     // leader, bit i: of pfix[i]
    bool ok = true;
    for (int tile = cluster; ok && tile < total_tiles && !*abort_flag; tile += nclusters) {
      const Tile t = decode_w(s, g, tile);
      const int nkb = w_kblocks<WK>(t);
      for (int kb = 0; kb < nkb; ++kb) {
        const int valid = w_kvalid<WK>(t, kb);
        if (fix_block(valid)) {
          int w_ok = 1;
          if (lane == 0)
            w_ok = mbar_wait(&s.landed[stage], (landed_phase >> stage) & 1u, abort_flag) ? 1 : 0;
          landed_phase ^= 1u << stage;
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
            ok = false;
            break;
          }
          const int nrow = ((valid + 15) & ~15) - valid;
          for (int i = lane; i < 4 * nrow * 8; i += 32) {
            const int box = i / (nrow * 8), rem = i - box * nrow * 8;
            const int r = valid + rem / 8, c16 = rem & 7;
            uint8_t* base = box < 2 ? s.a[stage] + box * WBOX : s.b[stage] + (box - 2) * WBOX;
            *reinterpret_cast<uint4*>(base + r * 128 + c16 * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (rank != 0) {
              mbar_arrive_release_cluster(mapa_shared(smem_u32(&s.pfix[stage]), 0));
            } else {
              w_ok = mbar_wait_acq_cluster(&s.pfix[stage], (pfix_phase >> stage) & 1u, abort_flag)
                         ? 1 : 0;
              if (w_ok) mbar_arrive(&s.full[stage]);
            }
          }
          pfix_phase ^= 1u << stage;
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
            ok = false;
            break;
          }
        }
        if (++stage == STAGES) stage = 0;
      }
    }
  } else {
    // ---- epilogue (both CTAs, warps 2..9): this CTA's 128 weight rows of the tile ---------
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    float (*stg)[32] = s.stg[warp - 2];
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < total_tiles; tile += nclusters) {
      const Tile t = decode_w(s, g, tile);
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(&s.tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + 128 * h);
      // the warp's 128 columns in two batches of 64, each in flight at once with one wait;
      // the accumulator goes back to the MMA before the second batch's stores
      const int row_base = t.mt * WBM + static_cast<int>(rank) * 128 + q * 32;
      float* out = static_cast<float*>(g.out) + (size_t)t.e * g.out_expert;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t v[2][32];
        tmem_ld_32x32b_x32(tbase + 64 * b, v[0]);
        tmem_ld_32x32b_x32(tbase + 64 * b + 32, v[1]);
        tmem_ld_wait();
        if (b == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[acc]), 0));
        }
#pragma unroll
        for (int i = 0; i < 2; ++i)
          store_f32_32(stg, lane, v[i], out, g.ld_out, row_base, g.m_valid,
                       t.nt * BN + 128 * h + 64 * b + 32 * i, g.n_valid);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  if (*abort_flag) {
    set_status(g.status, MOE_ERR_TIMEOUT);
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Cluster-of-two launch: as many clusters as fit at once (cached per device).
template <int WK>
int launch_wgrad_pair(const CUtensorMap& ma, const CUtensorMap& mb, const BwdArgs& g,
                      int sm_count, cudaStream_t st) {
  constexpr size_t smem = sizeof(WSmem<WK>) + 1024;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  static std::mutex mu;
  static int clusters_of[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return MOE_ERR_CUDA;
  if (cudaFuncSetAttribute(k_bwd_wgrad_pair<WK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  int nclusters;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (clusters_of[dev] == 0) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(sm_count & ~1);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_bwd_wgrad_pair<WK>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      clusters_of[dev] = n;
    }
    nclusters = clusters_of[dev];
  }
  if (nclusters > sm_count / 2) nclusters = sm_count / 2;
  if (launch_kernel(k_bwd_wgrad_pair<WK>, 2 * nclusters, kThreads, smem, st, 2, ma, mb, g) !=
      cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  count_launch();
  return MOE_OK;
}

}  // namespace

int launch_bwd_gemms(const void* dy, const void* gu, const void* h, const void* x_perm,
                     const int32_t* offsets, const void* w_gate_up, const void* w_down,
                     void* dgu, float* dx_perm, float* d_gate_up, float* d_down, int T, int H,
                     int I, int n_ffn, int K, int* status, int sm_count, cudaStream_t st) {
  const uint64_t rows = (uint64_t)T * K + BM;          // row buffers' allocation rows
  CUtensorMap m_dy128, m_dy64, m_dgu128, m_dgu64, m_h64, m_x64, m_wd, m_wgu;
  int rc;
  if ((rc = make_tma_map_bf16(&m_dy128, dy, rows, H, 128)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_dy64, dy, rows, H, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_dgu128, dgu, rows, 2ull * I, 128)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_dgu64, dgu, rows, 2ull * I, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_h64, h, rows, I, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_x64, x_perm, rows, H, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_wd, w_down, (uint64_t)n_ffn * H, I, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_wgu, w_gate_up, (uint64_t)n_ffn * 2 * I, H, 64)) != MOE_OK)
    return rc;

  BwdArgs g{};
  g.n_ffn = n_ffn;
  g.offsets = offsets;
  g.status = status;
  g.I = I;
  g.gu = static_cast<const __nv_bfloat16*>(gu);
  // dh = dy . W_d[e] (+ SwiGLU backward) -> dgu, then dx_perm = dgu . W_gu[e]: on the
  // CTA-pair kernel where the forward uses it
  const bool pair = dgrad_use_pair(T);
  if (pair) {
    if ((rc = launch_dgrad_pair(0, dy, H, w_down, H, I, gu, dgu, offsets, T, K, n_ffn, status,
                                sm_count, st)) != MOE_OK)
      return rc;
    if ((rc = launch_dgrad_pair(1, dgu, 2 * I, w_gate_up, 2 * I, H, nullptr, dx_perm, offsets, T,
                                K, n_ffn, status, sm_count, st)) != MOE_OK)
      return rc;
  }
  g.mode = kDH;
  g.kblocks = H / BK;
  g.n_tiles = (I + BN - 1) / BN;
  g.b_krows = H;
  g.n_valid = I;
  g.out = dgu;
  if (!pair && (rc = launch(m_dy128, m_wd, g, sm_count, st)) != MOE_OK) return rc;
  g.mode = kDX;
  g.kblocks = 2 * I / BK;
  g.n_tiles = (H + BN - 1) / BN;
  g.b_krows = 2 * I;
  g.n_valid = H;
  g.ld_out = H;
  g.out = dx_perm;
  if (!pair && (rc = launch(m_dgu128, m_wgu, g, sm_count, st)) != MOE_OK) return rc;
  // d_down[e] = dy^T h, then d_gate_up[e] = dgu^T x_perm: on CTA pairs (256 weight rows
  // per tile) unless MOE_TUNE_BWD_PAIR is 0 or 2
  const bool wpair = tuning(MOE_TUNE_BWD_PAIR) == 1 && sm_count >= 2;
  const int bm = wpair ? WBM : BM;
  g.mode = kDW;
  g.m_group = (int)tuning(MOE_TUNE_BWD_WGRAD_GROUP);
  g.mix_rows = (int)tuning(MOE_TUNE_BWD_WGRAD_MIX);
  g.m_valid = H;
  g.m_tiles = (H + bm - 1) / bm;
  g.n_tiles = (I + BN - 1) / BN;
  g.n_valid = I;
  g.ld_out = I;
  g.out_expert = (long long)H * I;
  g.out = d_down;
  // K rows per stage of the pair kernel: 64 (boxes of 64 rows) or 128
  const bool wk128 = wpair && tuning(MOE_TUNE_BWD_WGRAD_BK) == 128;
  CUtensorMap m_h128, m_x128;
  if (wk128 && ((rc = make_tma_map_bf16(&m_h128, h, rows, I, 128)) != MOE_OK ||
                (rc = make_tma_map_bf16(&m_x128, x_perm, rows, H, 128)) != MOE_OK))
    return rc;
  rc = wk128  ? launch_wgrad_pair<128>(m_dy128, m_h128, g, sm_count, st)
       : wpair ? launch_wgrad_pair<64>(m_dy64, m_h64, g, sm_count, st)
               : launch(m_dy64, m_h64, g, sm_count, st);
  if (rc != MOE_OK) return rc;
  g.m_valid = 2 * I;
  g.m_tiles = (2 * I + bm - 1) / bm;
  g.n_tiles = (H + BN - 1) / BN;
  g.n_valid = H;
  g.ld_out = H;
  g.out_expert = 2LL * I * H;
  g.out = d_gate_up;
  return wk128  ? launch_wgrad_pair<128>(m_dgu128, m_x128, g, sm_count, st)
         : wpair ? launch_wgrad_pair<64>(m_dgu64, m_x64, g, sm_count, st)
                 : launch(m_dgu64, m_x64, g, sm_count, st);
}

int launch_bwd_router_gemms(const void* dl3, int Tp, const void* x, const void* wr16,
                            const int32_t* offs_k, const int32_t* offs_m, int T, int E, int H,
                            float* d_router, float* dx, int* status, int sm_count,
                            cudaStream_t st) {
  CUtensorMap m_dl64, m_dl128, m_x64, m_wr64;
  int rc;
  if ((rc = make_tma_map_bf16(&m_dl64, dl3, 3ull * Tp, E, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_dl128, dl3, 3ull * Tp, E, 128)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_x64, x, (uint64_t)T, H, 64)) != MOE_OK) return rc;
  if ((rc = make_tma_map_bf16(&m_wr64, wr16, (uint64_t)E, H, 64)) != MOE_OK) return rc;
  BwdArgs g{};
  g.n_ffn = 1;
  g.status = status;
  // d_router [E, H] = sum over the three parts p and tokens t of dL_p[t]^T x[t]: one group
  // of 3 Tp K-rows (part p at rows [p Tp, p Tp + T)), x's row = K row mod Tp
  g.mode = kDW;
  g.offsets = offs_k;
  g.m_valid = E;
  g.m_tiles = (E + BM - 1) / BM;
  g.n_tiles = (H + BN - 1) / BN;
  g.n_valid = H;
  g.ld_out = H;
  g.out_expert = 0;
  g.b_kwrap = Tp;
  g.out = d_router;
  if ((rc = launch(m_dl64, m_x64, g, sm_count, st)) != MOE_OK) return rc;
  // dx [T, H] = dL_hi . W_r (bf16 operands): one group of T rows, K = E
  g = BwdArgs{};
  g.n_ffn = 1;
  g.status = status;
  g.mode = kDX;
  g.offsets = offs_m;
  g.kblocks = (E + BK - 1) / BK;
  g.n_tiles = (H + BN - 1) / BN;
  g.b_krows = 0;
  g.n_valid = H;
  g.ld_out = H;
  g.out = dx;
  return launch(m_dl128, m_wr64, g, sm_count, st);
}

}  // namespace moe
