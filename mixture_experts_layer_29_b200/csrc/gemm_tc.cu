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
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 48 KB
constexpr int kEpiWarps = 8;                         // two per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;           // producer, MMA, epilogue
constexpr int kMaxExperts = 1024;
constexpr uint32_t kTmemCols = 512;                  // two 256-column fp32 accumulators
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN);


// kDgradDH / kDgradDX: the backward's dgrad GEMMs on the CTA-pair kernel, B read MN-major
// (dh = dy . W_d[e] with the SwiGLU backward in the epilogue; dx rows = [dG | dU] . W_gu[e])
enum Mode : int {
  kGateUp = 0, kDownStore = 1, kDownAtomic = 2, kLogits = 3, kDgradDH = 4, kDgradDX = 5
};

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
  // router logits: each epilogue warp turns 32 rows x 16 columns around here so that its
  // global stores cover whole 64-byte row segments (row stride 20 floats: 16-byte aligned
  // and conflict-free for the row-wise float4 writes)
  alignas(16) float epi_stage[kEpiWarps][32][20];
};
static_assert(offsetof(SharedStorage, epi_stage) % 16 == 0, "16-byte staging rows");
static_assert(offsetof(SharedStorage, a) % 1024 == 0 && offsetof(SharedStorage, b) % 1024 == 0,
              "128-byte-swizzled TMA boxes need 1024-byte alignment");

struct GemmArgs {
  int mode;
  int n_ffn;
  int kblocks;        // K / 64
  int n_tiles;        // N tiles per M tile
  int b_rows;         // B rows per expert: 2I (gate/up) or H (down); 0 for the router
  int b_second;       // row offset of the second 128-row B box: I (gate/up) or 128
  int n_valid;        // valid output columns: I (h), H (y) or E (logits)
  int ld_out;         // output row length in elements
  const int32_t* offsets;
  void* out;
  const int32_t* perm_token;
  const float* row_gate;
  float scale;
  int* status;
  int a_kwrap;              // A's K coordinate wraps every a_kwrap k-blocks (0: no wrap)
  int dense_rows;           // > 0: one dense group of this many rows, offsets unused
  int ksplit;               // K splits per output tile (each writes its own fp32 slice)
  int kb_per_split;         // k-blocks per split
  int kchunk;               // k-blocks per tensor-core accumulation (0: the whole split)
  long long split_stride;   // elements between the outputs of consecutive splits
  const int32_t* gather_tok;  // non-null: A row r is row gather_tok[r] of A's tensor
  ZeroSpec zero;              // buffers cleared after the dependency wait
  int gu_raw;                 // gate/up: store G and U (bf16, [rows, 2I]) instead of h
  int logit_n;                // router: N tile (128, 192 or 256 logits)
  int half_tiles;             // pair kernel: an expert's last tile of <= 128 rows runs as M = 128
  void* gu_out;               // gate/up: also store G and U (bf16, [rows, 2I]) beside h, or null
  const __nv_bfloat16* gu_in; // kDgradDH: G | U of the rows ([rows, 2I], I = n_valid)
  int test_stall;             // testing (MOE_TUNE_TEST_STALL): tile 0 leaves its first
                              // k-block unloaded, so the waits on that stage run out
  int band;                   // pair kernel: M tiles per band of the tile order (1: M-major)
  int interleave;             // pair kernel: spread single-tile experts' tiles (see below)
  int a_trim;                 // pair kernel: load only the A rows of the group (a_box_rows)
  int swap_ab;                // pair kernel, forward: tiles of <= 128 rows run swapped (swap_npad)
  int stream_hint;            // pair kernel: single-tile experts' weights loaded evict-first
  int prefetch;               // pair kernel: L2 prefetch of the boxes this many k-blocks ahead
  int row_split;              // 0: every row of each expert; 1: its pair rows only (pair
                              // kernel); 2: the rest of them (one-CTA kernel): see pair_rows
};

// The rows of an expert's group that the CTA-pair GEMM takes when the forward is split
// between the two kernels (GemmArgs::row_split): whole 256-row tiles, plus the last partial
// tile when it holds more than 128 rows. The rest, at most 128 rows (a small expert, or a
// large expert's tail), goes to the one-CTA kernel as one 128-row tile: a pair tile of few
// rows holds two SMs for as long as a full one, the one-CTA tile holds one.
__device__ __forceinline__ int pair_rows(int count) {
  const int r = count & 255;
  return r <= 128 ? count - r : count;
}

// The testing hook of GemmArgs::test_stall: this (tile, k-block) is not loaded.
__device__ __forceinline__ bool stalled_stage(const GemmArgs& g, int tile, int kb, int kb0) {
  return g.test_stall != 0 && tile == 0 && kb == kb0;
}

struct Tile {
  int e, row0, row_end, nt, kb0, kb1, split;
};

__device__ __forceinline__ Tile decode_tile(const SharedStorage& s, const GemmArgs& g, int tile) {
  Tile t;
  const int per_split = s.toff[g.n_ffn] * g.n_tiles;
  t.split = tile / per_split;
  tile -= t.split * per_split;
  t.kb0 = t.split * g.kb_per_split;
  t.kb1 = min(g.kblocks, t.kb0 + g.kb_per_split);
  const int mt = tile / g.n_tiles;
  t.nt = tile - mt * g.n_tiles;
  // largest e with toff[e] <= mt (empty groups share the next group's toff and are skipped)
  int lo = 0, hi = g.n_ffn - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.toff[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  t.e = lo;
  const int begin = g.row_split == 2 ? s.offs[lo] + pair_rows(s.offs[lo + 1] - s.offs[lo]) : s.offs[lo];
  t.row0 = begin + (mt - s.toff[lo]) * BM;
  t.row_end = s.offs[lo + 1];
  return t;
}

__device__ __forceinline__ int chunk_len(const GemmArgs& g, const Tile& t) {
  return g.kchunk > 0 ? g.kchunk : (t.kb1 - t.kb0);
}

__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// ---- epilogue pieces of the expert GEMMs (one thread = one TMEM lane = one row) ---------
// gate/up: 32 columns of h = silu(G) * U from the gate accumulator columns at tbase + gcol
// and the up columns at tbase + ucol; h columns [oc, oc + 32) of the tile's 128.
// KEEP: whether G and U are also stored for the backward: 0 never, 1 always, 2 when
// g.gu_out is set (checked at run time).
template <int KEEP>
__device__ __forceinline__ void epi_gateup_chunk(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                                 int row, int gcol, int ucol, int oc) {
  uint32_t gr[32], ur[32];
  tmem_ld_32x32b_x32(tbase + gcol, gr);
  tmem_ld_32x32b_x32(tbase + ucol, ur);
  tmem_ld_wait();
  if (row >= t.row_end) return;
  if (g.gu_raw) {
    // G to columns [nt*128 + oc, +32) and U to I + that of the row (ld_out = 2I)
    __nv_bfloat16* base = static_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.ld_out + t.nt * BM + oc;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t* src = half ? ur : gr;
      uint4* dst = reinterpret_cast<uint4*>(base + (half ? g.n_valid : 0));
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = pack_bf16x2(__uint_as_float(src[v * 8 + 2 * i]), __uint_as_float(src[v * 8 + 2 * i + 1]));
        dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) +
                                        (size_t)row * g.ld_out + t.nt * BM + oc);
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
  if (KEEP == 1 || (KEEP == 2 && g.gu_out)) {
    // the same G and U, rounded to bf16 as the raw store rounds them, for the backward
    __nv_bfloat16* base = static_cast<__nv_bfloat16*>(g.gu_out) + (size_t)row * 2 * g.n_valid +
                          t.nt * BM + oc;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const uint32_t* src = part ? ur : gr;
      uint4* gdst = reinterpret_cast<uint4*>(base + (part ? g.n_valid : 0));
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = pack_bf16x2(__uint_as_float(src[v * 8 + 2 * i]),
                             __uint_as_float(src[v * 8 + 2 * i + 1]));
        gdst[v] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// down: 32 columns of y from the accumulator columns at tbase + tcol; output columns
// [oc, oc + 32) of the tile's 256. Deterministic store: through the warp's staging rows
// stg (32 x 80 bytes), so that a warp store covers 8 rows x 64 bytes; fused: s * g * y
// added to the token's fp32 accumulator (tok, sc of this row), through the same staging
// rows. Every lane of the warp must call it (warp shuffles and syncs).
__device__ __forceinline__ void epi_down_chunk(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                               int row, int tcol, int oc, int tok, float sc,
                                               float (*stg)[20], int lane) {
  uint32_t yr[32];
  tmem_ld_32x32b_x32(tbase + tcol, yr);
  tmem_ld_wait();
  const int col = t.nt * BN + oc;
  if (g.mode == kDownStore) {
    // this lane's row as 64 bytes of bf16 into the staging row, then 16 bytes per lane of
    // rows 8i + lane/4 out to global memory
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = v * 8 + i * 2;
        w[i] = pack_bf16x2(__uint_as_float(yr[j]), __uint_as_float(yr[j + 1]));
      }
      *reinterpret_cast<uint4*>(&stg[lane][4 * v]) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncwarp();
    if (col < g.n_valid) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 8 * i + (lane >> 2), ch = lane & 3;
        const int grow = row - lane + r;
        if (grow < t.row_end)
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) +
                                    (size_t)grow * g.ld_out + col + 8 * ch) =
              *reinterpret_cast<const uint4*>(&stg[r][4 * ch]);
      }
    }
    __syncwarp();
    return;
  }
  // fused: s * g * y of this lane's row into its token's fp32 accumulator, 16 columns at a
  // time through the staging rows, so that an atomic instruction covers 8 rows x 64
  // contiguous bytes (8 half lines) instead of 32 rows x 16 bytes (32 lines)
  const int valid = row < t.row_end ? 1 : 0;
#pragma unroll
  for (int h16 = 0; h16 < 2; ++h16) {
#pragma unroll
    for (int v = 0; v < 4; ++v)
      *reinterpret_cast<float4*>(&stg[lane][4 * v]) =
          make_float4(sc * __uint_as_float(yr[16 * h16 + 4 * v + 0]),
                      sc * __uint_as_float(yr[16 * h16 + 4 * v + 1]),
                      sc * __uint_as_float(yr[16 * h16 + 4 * v + 2]),
                      sc * __uint_as_float(yr[16 * h16 + 4 * v + 3]));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 8 * i + (lane >> 2), ch = lane & 3;
      const int tok_r = __shfl_sync(0xffffffffu, tok, r);
      const int ok_r = __shfl_sync(0xffffffffu, valid, r);
      const int c = col + 16 * h16 + 4 * ch;
      if (ok_r && c < g.n_valid)
        atomicAdd(reinterpret_cast<float4*>(static_cast<float*>(g.out) + (size_t)tok_r * g.ld_out + c),
                  *reinterpret_cast<const float4*>(&stg[r][4 * ch]));
    }
    __syncwarp();
  }
}

__device__ __forceinline__ void row_scale(const GemmArgs& g, const Tile& t, int row, int& tok,
                                          float& sc) {
  tok = 0;
  sc = 0.f;
  if (g.mode == kDownAtomic && row < t.row_end) {
    tok = g.perm_token[row];
    sc = g.scale * g.row_gate[row];
  }
}

// dgrad dh: 32 columns of dh at TMEM column tcol for this thread's row, output columns
// [oc, oc + 32) of the tile: dG, dU from the row's G and U (bf16), stored to [dG | dU].
__device__ __forceinline__ void epi_dh_chunk(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                             int row, int tcol, int oc) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(tbase + tcol, v);
  tmem_ld_wait();
  const int col = t.nt * BN + oc;
  if (row >= t.row_end || col >= g.n_valid) return;
  const int I = g.n_valid;
  const __nv_bfloat16* gr = g.gu_in + (size_t)row * 2 * I + col;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.out) + (size_t)row * 2 * I + col;
#pragma unroll
  for (int q8 = 0; q8 < 4; ++q8) {
    const uint4 G4 = *reinterpret_cast<const uint4*>(gr + 8 * q8);
    const uint4 U4 = *reinterpret_cast<const uint4*>(gr + I + 8 * q8);
    const __nv_bfloat16* Gb = reinterpret_cast<const __nv_bfloat16*>(&G4);
    const __nv_bfloat16* Ub = reinterpret_cast<const __nv_bfloat16*>(&U4);
    float dG[8], dU[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      swiglu_backward(__bfloat162float(Gb[i]), __bfloat162float(Ub[i]),
                      __uint_as_float(v[8 * q8 + i]), dG[i], dU[i]);
    *reinterpret_cast<uint4*>(dst + 8 * q8) =
        make_uint4(pack_bf16x2(dG[0], dG[1]), pack_bf16x2(dG[2], dG[3]),
                   pack_bf16x2(dG[4], dG[5]), pack_bf16x2(dG[6], dG[7]));
    *reinterpret_cast<uint4*>(dst + I + 8 * q8) =
        make_uint4(pack_bf16x2(dU[0], dU[1]), pack_bf16x2(dU[2], dU[3]),
                   pack_bf16x2(dU[4], dU[5]), pack_bf16x2(dU[6], dU[7]));
  }
}

// dgrad dx rows: 32 fp32 columns at TMEM column tcol, output columns [oc, oc + 32) of the
// tile, through the warp's staging rows (16 columns at a time) so that a warp store covers
// 8 rows x 64 bytes; rows past the expert's group are not stored.
__device__ __forceinline__ void epi_dx_chunk(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                             int row, int tcol, int oc, float (*stg)[20],
                                             int lane) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(tbase + tcol, v);
  tmem_ld_wait();
  float* out = static_cast<float*>(g.out);
  const int row_base = row - lane;
#pragma unroll
  for (int h16 = 0; h16 < 2; ++h16) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(&stg[lane][4 * i]) = make_float4(
          __uint_as_float(v[16 * h16 + 4 * i]), __uint_as_float(v[16 * h16 + 4 * i + 1]),
          __uint_as_float(v[16 * h16 + 4 * i + 2]), __uint_as_float(v[16 * h16 + 4 * i + 3]));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 8 * i + (lane >> 2);
      const int c = t.nt * BN + oc + 16 * h16 + 4 * (lane & 3);
      if (row_base + r < t.row_end && c < g.n_valid)
        *reinterpret_cast<float4*>(out + (size_t)(row_base + r) * g.ld_out + c) =
            *reinterpret_cast<const float4*>(&stg[r][4 * (lane & 3)]);
    }
    __syncwarp();
  }
}

// Epilogue of one 128 x 256 accumulator of the one-CTA kernel for one thread: its TMEM
// lane (row) and its half of the columns. The B tile is [128 gate rows | 128 up rows]
// (gate/up) or 256 rows of W_d (down): gate/up half h makes h columns [64h, 64h + 64)
// from gate columns [64h, 64h + 64) and up columns 128 + [64h, 64h + 64); down half h
// stores columns [128h, 128h + 128).
template <int KEEP>
__device__ __forceinline__ void epilogue_expert(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                                int row, int half, float (*stg)[20], int lane) {
  if (g.mode == kGateUp) {
#pragma unroll 1
    for (int c = 64 * half; c < 64 * half + 64; c += 32)
      epi_gateup_chunk<KEEP>(g, t, tbase, row, c, BM + c, c);
    return;
  }
  int tok;
  float sc;
  row_scale(g, t, row, tok, sc);
#pragma unroll 1
  for (int c = 128 * half; c < 128 * half + 128; c += 32)
    epi_down_chunk(g, t, tbase, row, c, c, tok, sc, stg, lane);
}

// LOGITS: the router instantiations (mode kLogits, running sums in the epilogue), with N
// tiles of NL logits; the expert GEMMs use <false, BN>.
template <bool LOGITS, int NL>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  SharedStorage& s = *reinterpret_cast<SharedStorage*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();

  // ---- set-up (no global memory before the dependency wait) ----------------------------
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
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
  g.zero.run(blockIdx.x, gridDim.x, threadIdx.x, kThreads);
  // tile table: toff[e] = sum_{e' < e} ceil(count_e' / 128)
  if (g.dense_rows > 0) {
    if (threadIdx.x == 0) {
      s.offs[0] = 0;
      s.offs[1] = g.dense_rows;
    }
  } else {
    for (int i = threadIdx.x; i <= g.n_ffn; i += kThreads) s.offs[i] = g.offsets[i];
  }
  __syncthreads();
  if (warp == 2) {
    const int per = (g.n_ffn + 31) / 32;
    const int b = lane * per;
    int local = 0;
    // M tiles of expert e: all of its rows, or (row_split == 2) the rows the pair kernel leaves
    auto tiles_of = [&](int e) {
      int rows = s.offs[e + 1] - s.offs[e];
      if (g.row_split == 2) rows -= pair_rows(rows);
      return (rows + BM - 1) / BM;
    };
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) local += tiles_of(b + i);
    const int inc = warp_inclusive_scan(local);
    int run = inc - local;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        s.toff[b + i] = run;
        run += tiles_of(b + i);
      }
    if (lane == 31) s.toff[g.n_ffn] = inc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = s.toff[g.n_ffn] * g.n_tiles * g.ksplit;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0 && g.gather_tok != nullptr) {
    // ---- TMA producer, gathered A: lane i fetches rows 4i..4i+3 of the A tile ----------
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles && !*abort_flag; tile += gridDim.x) {
      const Tile t = decode_tile(s, g, tile);
      int r[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)   // rows past the group repeat its last token (never stored)
        r[j] = g.gather_tok[min(t.row0 + 4 * lane + j, t.row_end - 1)];
      const int brow0 = t.e * g.b_rows + t.nt * (g.mode == kGateUp ? BM : BN);
      const int brow1 = brow0 + g.b_second;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const bool stall = stalled_stage(g, tile, kb, t.kb0);
        int w_ok = 1;
        if (lane == 0) {
          w_ok = mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag) ? 1 : 0;
          if (w_ok && !stall) mbar_arrive_expect_tx(&s.full[stage], STAGE_BYTES);
        }
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const int ka = g.a_kwrap > 0 ? kb % g.a_kwrap : kb;
        if (!stall) {
          tma_gather4(s.a[stage] + lane * 4 * (BK * 2), &tmA, ka * BK, r[0], r[1], r[2], r[3],
                      &s.full[stage]);
          if (lane == 0) {
            tma_load_2d(s.b[stage], &tmB, kb * BK, brow0, &s.full[stage]);
            tma_load_2d(s.b[stage] + B_BYTES / 2, &tmB, kb * BK, brow1, &s.full[stage]);
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 0) {
    // ---- TMA producer ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const Tile t = decode_tile(s, g, tile);
        const int brow0 = t.e * g.b_rows + t.nt * (LOGITS ? NL : g.mode == kGateUp ? BM : BN);
        const int brow1 = brow0 + g.b_second;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) break;
          if (!stalled_stage(g, tile, kb, t.kb0)) {
            mbar_arrive_expect_tx(&s.full[stage], LOGITS ? A_BYTES + NL * BK * 2 : STAGE_BYTES);
            const int ka = g.a_kwrap > 0 ? kb % g.a_kwrap : kb;
            tma_load_2d(s.a[stage], &tmA, ka * BK, t.row0, &s.full[stage]);
            tma_load_2d(s.b[stage], &tmB, kb * BK, brow0, &s.full[stage]);
            if (!LOGITS || NL == 256)
              tma_load_2d(s.b[stage] + B_BYTES / 2, &tmB, kb * BK, brow1, &s.full[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: one TMEM accumulator per chunk of k-blocks -------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const Tile t = decode_tile(s, g, tile);
        const int cl = chunk_len(g, t);
        for (int c0 = t.kb0; ok && c0 < t.kb1; c0 += cl) {
          const int c1 = min(c0 + cl, t.kb1);
          if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
          for (int kb = c0; kb < c1; ++kb) {
            if (!mbar_wait(&s.full[stage], phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(s.a[stage]);
            const uint32_t b0 = smem_u32(s.b[stage]);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16(d_tmem, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32),
                        LOGITS ? idesc_bf16_f32(BM, NL) : kIdesc, (kb > c0 || k > 0) ? 1u : 0u);
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
    }
  } else {
    // ---- epilogue (warps 2..9): TMEM lane quarter = warp % 4, column half = (warp-2) / 4
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      const Tile t = decode_tile(s, g, tile);
      const int row = t.row0 + row_in_tile;
      const int cl = chunk_len(g, t);
      constexpr int NH = NL / 2;     // router: columns per thread (half of the tile)
      float sum[LOGITS ? NH : 1];    // router logits: running fp32 sum of this half-row
      if constexpr (LOGITS) {
#pragma unroll
        for (int i = 0; i < NH; ++i) sum[i] = 0.f;
      }
      for (int c0 = t.kb0; c0 < t.kb1; c0 += cl) {
        // one lane waits, the warp follows it: tcgen05.ld below needs all 32 lanes
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(&s.tfull[acc], acc_phase, abort_flag) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * BN);
        if constexpr (LOGITS) {
          // add this chunk to the running sum (fp32, round to nearest)
#pragma unroll
          for (int c = 0; c < NH; c += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + NH * half + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) sum[c + i] = __fadd_rn(sum[c + i], __uint_as_float(v[i]));
          }
        } else {
          epilogue_expert<2>(g, t, tbase, row, half, s.epi_stage[warp - 2], lane);
        }
        tc_fence_before();
        mbar_arrive(&s.tempty[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if constexpr (LOGITS) {
        if (ok) {
          // 32 rows x 16 columns at a time through shared memory: lane l then stores
          // row 8i + l/4, columns 4(l%4)..+3, so a warp store covers 8 rows x 64 bytes
          float (*stg)[20] = s.epi_stage[warp - 2];
          float* outp = static_cast<float*>(g.out) + t.split * g.split_stride;
          const int col0 = t.nt * NL + NH * half;
          const bool vec = (g.ld_out & 3) == 0 && (reinterpret_cast<uintptr_t>(g.out) & 15) == 0;
#pragma unroll
          for (int c = 0; c < NH; c += 16) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<float4*>(&stg[lane][4 * v]) =
                  make_float4(sum[c + 4 * v], sum[c + 4 * v + 1], sum[c + 4 * v + 2],
                              sum[c + 4 * v + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 8 * i + (lane >> 2), cc = 4 * (lane & 3);
              const float4 val = *reinterpret_cast<const float4*>(&stg[r][cc]);
              const int grow = t.row0 + q * 32 + r;
              const int gcol = col0 + c + cc;
              if (grow < t.row_end) {
                float* d = outp + (size_t)grow * g.ld_out + gcol;
                if (vec && gcol + 4 <= g.n_valid) {
                  *reinterpret_cast<float4*>(d) = val;
                } else {
                  const float vv[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    if (gcol + j < g.n_valid) d[j] = vv[j];
                }
              }
            }
            __syncwarp();
          }
        }
      }
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

// ---- CTA-pair variant of the expert GEMMs (tcgen05 cta_group::2) -------------------------
// A cluster of two CTAs computes a 256 x 256 tile: CTA r loads rows [128r, 128r+128) of the
// A tile and B rows [128r, 128r+128) of the N tile (gate/up: CTA 0 the gate rows, CTA 1
// the up rows), so each CTA moves 32 KB per k-block instead of 48 KB. Both CTAs' TMA loads
// count on the leader's (rank 0) full barrier; the leader's single thread issues
// tcgen05.mma.cta_group::2 (M = 256) and commits to the empty / accumulator-full barriers
// of both CTAs (two commits, one per CTA); both CTAs' epilogues read their own TMEM rows
// (the same column layout as the one-CTA kernel) and release the accumulator on the
// leader's barrier.
// Half tiles: an expert's last tile holds count mod 256 rows; when that is at most 128 it
// runs as an M = 128 MMA over both CTAs (64 rows each: A loaded from row0 + 64r, its first
// 64 rows used), which halves the tail's padded work. The accumulator then lands in TMEM
// columns [0, 128) as the 2 x 2 layout: lanes 0-63 hold the CTA's 64 rows for N columns
// [0, 128) (the leader's B rows), lanes 64-127 the same rows for N columns [128, 256) (the
// peer's B rows). So that each lane quarter holds gate and up columns of the same h
// columns, the gate/up half tile loads CTA r's B as gate rows [64r, 64r + 64) of the N tile
// followed by the same up rows (two 64-row boxes, the same shared-memory layout as one
// 128-row box); full tiles keep the 128-row gate / up boxes.
constexpr int BMP = 256;                             // M rows per CTA pair
constexpr int PSTAGES = 6;                           // 32 KB per stage per CTA
constexpr int P_B_BYTES = 128 * BK * 2;              // 16 KB: this CTA's half of B

struct alignas(1024) PairStorage {
  uint8_t a[PSTAGES][A_BYTES];
  uint8_t b[PSTAGES][P_B_BYTES];
  uint64_t full[PSTAGES];       // leader: both CTAs' bytes; peer: unused
  uint64_t empty[PSTAGES];      // both: the leader's MMA commit
  uint64_t tfull[2];            // both: the leader's MMA commit
  uint64_t tempty[2];           // leader: one arrival per epilogue warp of both CTAs
  uint32_t tmem_base;
  int abort_flag;
  int offs[kMaxExperts + 1];
  int toff[kMaxExperts + 1];    // prefix of ceil(count / 256) over the multi-tile experts
  int n_single;                 // experts of one M tile spread through the order (see below)
  int16_t single[kMaxExperts];  // those experts, in index order
  // deterministic down store (see epilogue_expert); read and written as 16-byte vectors
  alignas(16) float epi_stage[kEpiWarps][32][20];
};
static_assert(offsetof(PairStorage, epi_stage) % 16 == 0, "16-byte staging rows");
static_assert(offsetof(PairStorage, a) % 1024 == 0 && offsetof(PairStorage, b) % 1024 == 0,
              "128-byte-swizzled TMA boxes need 1024-byte alignment");

// End of expert e's rows in the CTA-pair kernel (its pair rows when the forward is split).
__device__ __forceinline__ int pair_end(const PairStorage& s, const GemmArgs& g, int e) {
  return g.row_split == 1 ? s.offs[e] + pair_rows(s.offs[e + 1] - s.offs[e]) : s.offs[e + 1];
}

// Tile order of the CTA-pair kernel. Tiles are handed out round-robin in this order, so
// the order is also roughly the time at which a tile runs.
//  * Experts of a single M tile (at most 256 rows; g.interleave) stream their whole weight
//    matrix for one tile each: their tiles are DRAM-bound, while the multi-tile experts'
//    tiles reuse each B tile over several M tiles and are bound by the tensor pipe. So the
//    single-tile experts' tiles ("S") are spread evenly through the others ("L"):
//    position i is an S tile when floor((i+1) TS / Ttot) > floor(i TS / Ttot), with TS S
//    tiles out of Ttot. Their weight streams then overlap the L tiles' MMAs instead of
//    filling whole waves with DRAM-bound tiles. S tiles go expert by expert, N fastest.
//  * L tiles: expert e owns L tiles [toff[e], toff[e+1]) * n_tiles. Inside an expert the
//    M tiles go in bands of g.band: a band's tiles run N tile by N tile, its M tiles
//    fastest. g.band = 1 is plain M-major order (N fastest).
__device__ __forceinline__ Tile decode_pair_tile(const PairStorage& s, const GemmArgs& g, int tile) {
  Tile t;
  t.split = 0;
  t.kb0 = 0;
  t.kb1 = g.kblocks;
  if (s.n_single > 0) {
    const long long ts = (long long)s.n_single * g.n_tiles;
    const long long tot = ts + (long long)s.toff[g.n_ffn] * g.n_tiles;
    const int ns0 = (int)((long long)tile * ts / tot);
    const int ns1 = (int)((long long)(tile + 1) * ts / tot);
    if (ns1 > ns0) {                                    // the ns0-th S tile
      const int k = ns0 / g.n_tiles;
      const int e = s.single[k];
      t.nt = ns0 - k * g.n_tiles;
      t.e = e;
      t.row0 = s.offs[e];
      t.row_end = pair_end(s, g, e);
      return t;
    }
    tile -= ns0;                                        // the tile-th L tile
  }
  const int mt_any = tile / g.n_tiles;
  int lo = 0, hi = g.n_ffn - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.toff[mid] <= mt_any) lo = mid; else hi = mid - 1;
  }
  int mt;
  if (g.band > 1) {
    const int l = tile - s.toff[lo] * g.n_tiles;       // tile within the expert
    const int per_band = g.band * g.n_tiles;
    const int j = l / per_band;
    const int o = l - j * per_band;
    const int h = min(g.band, s.toff[lo + 1] - s.toff[lo] - j * g.band);   // band height
    t.nt = o / h;
    mt = j * g.band + (o - t.nt * h);
  } else {
    mt = mt_any - s.toff[lo];
    t.nt = tile - mt_any * g.n_tiles;
  }
  t.e = lo;
  t.row0 = s.offs[lo] + mt * BMP;
  t.row_end = pair_end(s, g, lo);
  return t;
}

__device__ __forceinline__ bool half_tile(const GemmArgs& g, const Tile& t) {
  return g.half_tiles && t.row_end - t.row0 <= 128;
}

// Rows of CTA r's A box in a pair tile. The CTA's MMA rows are [row0 + per r, + per) with
// per = 64 (half tile) or 128; only those inside the expert's group are ever stored, so
// with g.a_trim only they are loaded: a box of 16, 64 or 128 rows, or nothing. The MMA
// reads whatever the rest of the A stage holds, and the rows it makes there are dropped.
// A single-row expert then moves 2 KB of A per k-block instead of 16 KB, which matters
// because such tiles are bound by how fast the SM fills its shared memory.
__device__ __forceinline__ int a_box_rows(const GemmArgs& g, const Tile& t, bool half, int r) {
  const int per = half ? 64 : 128;
  if (!g.a_trim) return 128;
  const int need = min(t.row_end - (t.row0 + per * r), per);
  return need <= 0 ? 0 : need <= 16 ? 16 : need <= 64 ? 64 : 128;
}

// Swap tiles (g.swap_ab, forward GEMMs). An M = 128 tile over the CTA pair (64 rows per
// CTA) costs the tensor pipe as many cycles as an M = 256 one, so a tile of few rows
// (small experts, an expert's tail) costs a full tile of MMA time. With the operands
// swapped the expert's weights are the M = 256 side and the tile's rows the N side,
// N = npad (16, 32, 64 or 128: the rows rounded up), and the MMA time shrinks with the
// rows: such a tile is bound by streaming its weights. CTA r then holds weight rows
// [128r, 128r + 128) of the N tile (gate/up: 64 gate rows and the same 64 up rows, as the
// half tiles load them) and rows [row0 + r npad/2, + npad/2) of the tile's rows.
// The accumulator is transposed: TMEM lane = output feature, column = row of the tile.
__device__ __forceinline__ int swap_npad(const GemmArgs& g, const Tile& t) {
  if (!g.swap_ab) return 0;
  const int rows = t.row_end - t.row0;
  if (rows > 128) return 0;
  return rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : 128;
}

// The pair kernel's 8 epilogue warps (256 threads) meet here; named barrier 1.
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Epilogue of a swap tile, for every epilogue thread of CTA `rank` (warp quarter q, column
// half h); all 8 epilogue warps take part (named barrier 1). Per 32 columns (rows of the
// tile): each warp moves 16 columns of its 32 lanes
// from TMEM into S[row][feature] (fp32, row stride 132 floats), then the 256 threads write
// whole output rows from S. TMEM lane l is output feature l of the CTA's 128: gate/up:
// h column nt * 128 + 64 rank + (l mod 64), from gate (l < 64) and up (l >= 64); down:
// output column nt * 256 + 128 rank + l. KEEP: as epi_gateup_chunk.
template <int KEEP>
__device__ __forceinline__ void epilogue_swap(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                              uint32_t rank, int q, int h, float* S, int npad) {
  constexpr int SS = 132;
  const int lane = threadIdx.x & 31;
  const int u = threadIdx.x - 64;                     // 0..255 over the epilogue warps
  // S spans every warp's staging rows: wait until all warps are done with the last tile
  epi_bar();
#pragma unroll 1
  for (int c0 = 0; c0 < npad; c0 += 32) {
    const int ncol = min(32, npad - c0);
    if (16 * h < ncol) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(tbase + (uint32_t)(c0 + 16 * h), v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) S[(16 * h + j) * SS + 32 * q + lane] = __uint_as_float(v[j]);
    }
    epi_bar();
    if (g.mode == kGateUp) {
      // 32 rows x 8 groups of 8 h columns: one 16-byte store of h (or of G and U)
      const int j = u >> 3, f8 = u & 7;
      const int row = t.row0 + c0 + j;
      if (j < ncol && row < t.row_end) {
        const float4* sg = reinterpret_cast<const float4*>(S + j * SS + 8 * f8);
        const float4* su = reinterpret_cast<const float4*>(S + j * SS + 64 + 8 * f8);
        const float4 g0 = sg[0], g1 = sg[1], u0 = su[0], u1 = su[1];
        const float G[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float U[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        const int col = t.nt * BM + 64 * (int)rank + 8 * f8;
        if (g.gu_raw) {
          __nv_bfloat16* base = static_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.ld_out + col;
          *reinterpret_cast<uint4*>(base) =
              make_uint4(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]),
                         pack_bf16x2(G[4], G[5]), pack_bf16x2(G[6], G[7]));
          *reinterpret_cast<uint4*>(base + g.n_valid) =
              make_uint4(pack_bf16x2(U[0], U[1]), pack_bf16x2(U[2], U[3]),
                         pack_bf16x2(U[4], U[5]), pack_bf16x2(U[6], U[7]));
        } else {
          float hv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) hv[i] = silu_f(G[i]) * U[i];
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.ld_out + col) =
              make_uint4(pack_bf16x2(hv[0], hv[1]), pack_bf16x2(hv[2], hv[3]),
                         pack_bf16x2(hv[4], hv[5]), pack_bf16x2(hv[6], hv[7]));
          if (KEEP == 1 || (KEEP == 2 && g.gu_out)) {
            __nv_bfloat16* base = static_cast<__nv_bfloat16*>(g.gu_out) +
                                  (size_t)row * 2 * g.n_valid + col;
            *reinterpret_cast<uint4*>(base) =
                make_uint4(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]),
                           pack_bf16x2(G[4], G[5]), pack_bf16x2(G[6], G[7]));
            *reinterpret_cast<uint4*>(base + g.n_valid) =
                make_uint4(pack_bf16x2(U[0], U[1]), pack_bf16x2(U[2], U[3]),
                           pack_bf16x2(U[4], U[5]), pack_bf16x2(U[6], U[7]));
          }
        }
      }
    } else if (g.mode == kDownStore) {
      // 32 rows x 16 groups of 8 output columns
#pragma unroll 1
      for (int it = u; it < 32 * 16; it += 256) {
        const int j = it >> 4, f8 = it & 15;
        const int row = t.row0 + c0 + j;
        const int col = t.nt * BN + 128 * (int)rank + 8 * f8;
        if (j < ncol && row < t.row_end && col < g.n_valid) {
          const float4* sy = reinterpret_cast<const float4*>(S + j * SS + 8 * f8);
          const float4 a = sy[0], b = sy[1];
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (size_t)row * g.ld_out + col) =
              make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                         pack_bf16x2(b.z, b.w));
        }
      }
    } else {
      // fused: s * g * y added into the token's fp32 accumulator, 4 columns at a time
#pragma unroll 1
      for (int it = u; it < 32 * 32; it += 256) {
        const int j = it >> 5, f4 = it & 31;
        const int row = t.row0 + c0 + j;
        const int col = t.nt * BN + 128 * (int)rank + 4 * f4;
        if (j < ncol && row < t.row_end && col < g.n_valid) {
          const int tok = g.perm_token[row];
          const float sc = g.scale * g.row_gate[row];
          const float4 y = *reinterpret_cast<const float4*>(S + j * SS + 4 * f4);
          atomicAdd(reinterpret_cast<float4*>(static_cast<float*>(g.out) + (size_t)tok * g.ld_out + col),
                    make_float4(sc * y.x, sc * y.y, sc * y.z, sc * y.w));
        }
      }
    }
    epi_bar();
  }
}

// Epilogue of one pair tile for one thread of warp quarter q and column half h. Full tile
// (M = 256): row 128r + 32q + lane, as in the one-CTA kernel. Half tile (M = 128): row
// 64r + 32(q & 1) + lane and N block ib = q >> 1; gate/up: h columns 64 ib + 32h + [0, 32)
// from the gate TMEM columns 32h + [0, 32) and the up columns 64 + 32h + [0, 32); down:
// output columns 128 ib + 64h + [0, 64) from TMEM columns 64h + [0, 64).
// Kinds of the CTA-pair kernel: the forward, the forward that also keeps G | U, and the
// backward's dgrad modes (B read MN-major); each its own instantiation.
constexpr int kPairFwd = 0, kPairFwdKeep = 1, kPairDgrad = 2;

template <int KIND>
__device__ __forceinline__ void epilogue_pair(const GemmArgs& g, const Tile& t, uint32_t tbase,
                                              uint32_t rank, int q, int h, float (*stg)[20],
                                              int lane) {
  if constexpr (KIND == kPairDgrad) {
    // full tile: row 128r + 32q + lane, columns [128h, 128h + 128); half tile: as the down
    // store below
    const bool half = half_tile(g, t);
    const int row = half ? t.row0 + 64 * (int)rank + 32 * (q & 1) + lane
                         : t.row0 + 128 * (int)rank + q * 32 + lane;
#pragma unroll 1
    for (int j = 0; j < (half ? 64 : 128); j += 32) {
      const int tcol = half ? 64 * h + j : 128 * h + j;
      const int oc = half ? 128 * (q >> 1) + 64 * h + j : 128 * h + j;
      if (g.mode == kDgradDH) epi_dh_chunk(g, t, tbase, row, tcol, oc);
      else epi_dx_chunk(g, t, tbase, row, tcol, oc, stg, lane);
    }
  } else {
    if (!half_tile(g, t)) {
      epilogue_expert<KIND == kPairFwdKeep ? 1 : 0>(g, t, tbase,
                                                     t.row0 + 128 * (int)rank + q * 32 + lane,
                                                     h, stg, lane);
      return;
    }
    const int row = t.row0 + 64 * (int)rank + 32 * (q & 1) + lane;
    const int ib = q >> 1;
    if (g.mode == kGateUp) {
      epi_gateup_chunk<KIND == kPairFwdKeep ? 1 : 0>(g, t, tbase, row, 32 * h, 64 + 32 * h,
                                                      64 * ib + 32 * h);
      return;
    }
    int tok;
    float sc;
    row_scale(g, t, row, tok, sc);
#pragma unroll 1
    for (int j = 0; j < 64; j += 32)
      epi_down_chunk(g, t, tbase, row, 64 * h + j, 128 * ib + 64 * h + j, tok, sc, stg, lane);
  }
}

// What the producer of CTA `rank` loads for a pair tile: its A box (rows and tensor map) and
// its B half (rows or, MN-major, columns).
struct PairPlan {
  int arow, a_rows, brow, bcol;
  bool split_b, stream;
  const CUtensorMap* a_map;
};

__device__ __forceinline__ PairPlan pair_plan(const PairStorage& s, const GemmArgs& g,
                                              const Tile& t, int rank, bool b_mn,
                                              const CUtensorMap* mA, const CUtensorMap* mA64,
                                              const CUtensorMap* mA32, const CUtensorMap* mA16,
                                              const CUtensorMap* mA8) {
  PairPlan p;
  const int npad = swap_npad(g, t);                  // swap tile: npad / 2 rows per CTA
  const bool half = !npad && half_tile(g, t);
  p.split_b = (half || npad) && g.mode == kGateUp;   // 64 gate + 64 up rows
  p.arow = npad ? t.row0 + (npad / 2) * rank : t.row0 + (half ? 64 : 128) * rank;
  p.brow = g.mode != kGateUp ? t.e * g.b_rows + t.nt * BN + 128 * rank
           : p.split_b ? t.e * g.b_rows + t.nt * BM + 64 * rank
                       : t.e * g.b_rows + rank * g.b_second + t.nt * BM;
  // MN-major B (dgrad): this CTA's 128 N columns as two 64 x 64 boxes of K rows
  p.bcol = t.nt * BN + 128 * rank;
  p.stream = g.stream_hint && !b_mn && s.offs[t.e + 1] - s.offs[t.e] <= BMP;
  p.a_rows = npad ? npad / 2 : a_box_rows(g, t, half, rank);
  p.a_map = p.a_rows == 128 ? mA : p.a_rows == 64 ? mA64 : p.a_rows == 32 ? mA32
          : p.a_rows == 16 ? mA16 : mA8;
  return p;
}

// The weight boxes pair_plan's loads read for k-block kb of a tile of a single-tile expert
// (p.stream), brought into L2 g.prefetch k-blocks ahead of the loads. Such tiles stream their
// weights from DRAM with six stages in flight and wait on DRAM latency; the other tiles find
// their operands in L2 and keep the SM's TMA unit busy, so they prefetch nothing.
__device__ __forceinline__ void pair_prefetch(const PairPlan& p, const GemmArgs& g, int kb,
                                              const CUtensorMap* mB, const CUtensorMap* mB64) {
  if (!p.stream) return;
  if (p.split_b) {
    tma_prefetch_2d(mB64, kb * BK, p.brow);
    tma_prefetch_2d(mB64, kb * BK, p.brow + g.b_second);
  } else {
    tma_prefetch_2d(mB, kb * BK, p.brow);
  }
}

// tmB64: the gate/up B tensor with 64-row boxes (half tiles); unused by the down GEMM.
// KIND: kPairFwd, kPairFwdKeep or kPairDgrad (see epilogue_pair), so that the plain
// forward carries none of the other kinds' code.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA64,
                        const __grid_constant__ CUtensorMap tmA32,
                        const __grid_constant__ CUtensorMap tmA16,
                        const __grid_constant__ CUtensorMap tmA8,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB64, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  PairStorage& s = *reinterpret_cast<PairStorage*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();            // 0: leader, 1: peer
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  pdl_launch_dependents();

  // ---- set-up (no global memory before the dependency wait) ----------------------------
  if (threadIdx.x == 0) {
    for (int i = 0; i < PSTAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 2 * kEpiWarps);
    }
    s.abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (g.half_tiles && g.mode == kGateUp) prefetch_tensormap(&tmB64);
    if (g.a_trim || g.swap_ab) {
      prefetch_tensormap(&tmA64);
      prefetch_tensormap(&tmA16);
    }
    if (g.swap_ab) {
      prefetch_tensormap(&tmA32);
      prefetch_tensormap(&tmA8);
    }
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
    // L tiles per expert (multi-tile experts, or all with g.interleave off) and the list
    // of single-tile experts; lane l takes a contiguous run of experts
    const int per = (g.n_ffn + 31) / 32;
    const int b = lane * per;
    int local = 0, nsingle = 0;
    auto tiles_of = [&](int e) {
      int rows = s.offs[e + 1] - s.offs[e];
      if (g.row_split == 1) rows = pair_rows(rows);
      return (rows + BMP - 1) / BMP;
    };
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        const int m = tiles_of(b + i);
        if (g.interleave && m == 1) ++nsingle;
        else local += m;
      }
    const int inc = warp_inclusive_scan(local);
    const int sinc = warp_inclusive_scan(nsingle);
    int run = inc - local, srun = sinc - nsingle;
    for (int i = 0; i < per; ++i)
      if (b + i < g.n_ffn) {
        s.toff[b + i] = run;
        const int m = tiles_of(b + i);
        if (g.interleave && m == 1) s.single[srun++] = (int16_t)(b + i);
        else run += m;
      }
    if (lane == 31) {
      s.toff[g.n_ffn] = inc;
      s.n_single = sinc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = (s.toff[g.n_ffn] + s.n_single) * g.n_tiles;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0) {
    // ---- TMA producer (both CTAs): this CTA's A rows and B half, counted on the leader --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t policy = l2_evict_first_policy();
      constexpr bool b_mn = KIND == kPairDgrad;
      const int pf = g.prefetch;
      for (int tile = cluster; tile < total_tiles && !*abort_flag; tile += nclusters) {
        const Tile t = decode_pair_tile(s, g, tile);
        const PairPlan p = pair_plan(s, g, t, (int)rank, b_mn, &tmA, &tmA64, &tmA32, &tmA16, &tmA8);
        const int npad = swap_npad(g, t);
        const bool half = !npad && half_tile(g, t);
        // the leader expects both CTAs' bytes: B halves of 16 KB and the two A boxes
        const uint32_t tx = 2 * P_B_BYTES +
            (npad ? (uint32_t)npad * BK * 2
                  : (uint32_t)(a_box_rows(g, t, half, 0) + a_box_rows(g, t, half, 1)) * BK * 2);
        // the cluster's next tile, for prefetches that run past this tile's last k-block
        const bool has_next = pf > 0 && tile + nclusters < total_tiles;
        Tile tn = t;
        PairPlan pn = p;
        if (has_next) {
          tn = decode_pair_tile(s, g, tile + nclusters);
          pn = pair_plan(s, g, tn, (int)rank, b_mn, &tmA, &tmA64, &tmA32, &tmA16, &tmA8);
        }
        if (pf > 0 && tile == cluster)
          for (int kb = 0; kb < pf && kb < g.kblocks; ++kb) pair_prefetch(p, g, kb, &tmB, &tmB64);
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag)) break;
          if (stalled_stage(g, tile, kb, 0)) {   // neither CTA loads; nothing is expected
            if (++stage == PSTAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&s.full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], tx);
          if (p.a_rows > 0) tma_load_2d_pair(s.a[stage], p.a_map, kb * BK, p.arow, full_leader);
          if (b_mn) {
            const int y = t.e * g.b_rows + kb * BK;
            tma_load_2d_pair(s.b[stage], &tmB, p.bcol, y, full_leader);
            tma_load_2d_pair(s.b[stage] + P_B_BYTES / 2, &tmB, p.bcol + 64, y, full_leader);
          } else if (p.stream) {
            // an expert of one M tile: its weights are read once, so they leave L2 first
            if (p.split_b) {
              tma_load_2d_pair_hint(s.b[stage], &tmB64, kb * BK, p.brow, full_leader, policy);
              tma_load_2d_pair_hint(s.b[stage] + P_B_BYTES / 2, &tmB64, kb * BK,
                                    p.brow + g.b_second, full_leader, policy);
            } else {
              tma_load_2d_pair_hint(s.b[stage], &tmB, kb * BK, p.brow, full_leader, policy);
            }
          } else if (p.split_b) {
            tma_load_2d_pair(s.b[stage], &tmB64, kb * BK, p.brow, full_leader);
            tma_load_2d_pair(s.b[stage] + P_B_BYTES / 2, &tmB64, kb * BK, p.brow + g.b_second,
                             full_leader);
          } else {
            tma_load_2d_pair(s.b[stage], &tmB, kb * BK, p.brow, full_leader);
          }
          if (pf > 0) {
            const int kp = kb + pf;
            if (kp < g.kblocks) pair_prefetch(p, g, kp, &tmB, &tmB64);
            else if (has_next && kp - g.kblocks < g.kblocks)
              pair_prefetch(pn, g, kp - g.kblocks, &tmB, &tmB64);
          }
          if (++stage == PSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (leader only) ---------------------------------------------------------
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total_tiles && !*abort_flag; tile += nclusters) {
        constexpr bool b_mn = KIND == kPairDgrad;
        const Tile mt = decode_pair_tile(s, g, tile);
        const int npad = swap_npad(g, mt);
        // swap tile: A = the weights (s.b), B = the tile's rows (s.a), N = npad
        const uint32_t idesc = npad ? idesc_bf16_f32(BMP, npad)
                                    : idesc_bf16_f32_major(half_tile(g, mt) ? 128 : BMP, BN,
                                                           false, b_mn);
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          if (npad) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(d_tmem, sw128_kmajor_desc(b0 + k * 32), sw128_kmajor_desc(a0 + k * 32),
                             idesc, (kb > 0 || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(d_tmem, sw128_kmajor_desc(a0 + k * 32),
                             b_mn ? sw128_mnmajor_desc(b0 + k * 2048, P_B_BYTES / 2)
                                  : sw128_kmajor_desc(b0 + k * 32),
                             idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          const uint32_t e_local = smem_u32(&s.empty[stage]);
          umma_commit_pair(mapa_shared(e_local, 0));
          umma_commit_pair(mapa_shared(e_local, 1));
          if (++stage == PSTAGES) {
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
  } else {
    // ---- epilogue (both CTAs, warps 2..9): this CTA's rows of the tile -------------------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < total_tiles; tile += nclusters) {
      const Tile t = decode_pair_tile(s, g, tile);
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(&s.tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      int npad = 0;
      if constexpr (KIND != kPairDgrad) npad = swap_npad(g, t);
      if (npad) {
        if constexpr (KIND != kPairDgrad)
          epilogue_swap<KIND == kPairFwdKeep ? 1 : 0>(g, t, tbase, rank, q, half,
                                                      &s.epi_stage[0][0][0], npad);
      } else {
        epilogue_pair<KIND>(g, t, tbase, rank, q, half, s.epi_stage[warp - 2], lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- tear-down ------------------------------------------------------------------------
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

// rows x cols bf16 matrix, row-major; box = 64 columns x box_rows rows (128 for tiled
// loads, 1 for four-row gathers), 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
             uint32_t box_rows = BM) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

int launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, int sm_count,
               cudaStream_t st) {
  constexpr size_t smem = sizeof(SharedStorage) + 1024;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  auto kern = g.mode != kLogits ? k_grouped_gemm_tc<false, BN>
               : g.logit_n == 128 ? k_grouped_gemm_tc<true, 128>
               : g.logit_n == 192 ? k_grouped_gemm_tc<true, 192>
                                  : k_grouped_gemm_tc<true, 256>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  const cudaError_t e = launch_kernel(kern, sm_count, kThreads, smem, st, 1, ma, mb, g);
  count_launch();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Cluster-of-two launch of the CTA-pair kernel: as many clusters as fit at once (cached
// per device), so the persistent tile loop never waits for a cluster slot.
// A's tensor with boxes of 128, 64, 32, 16 and 8 rows (see a_box_rows and swap_npad).
struct AMaps {
  CUtensorMap m128, m64, m32, m16, m8;
};
int make_amaps(AMaps* m, const void* base, uint64_t rows, uint64_t cols) {
  int rc;
  if ((rc = make_map(&m->m128, base, rows, cols, 128)) != MOE_OK ||
      (rc = make_map(&m->m64, base, rows, cols, 64)) != MOE_OK ||
      (rc = make_map(&m->m32, base, rows, cols, 32)) != MOE_OK ||
      (rc = make_map(&m->m16, base, rows, cols, 16)) != MOE_OK ||
      (rc = make_map(&m->m8, base, rows, cols, 8)) != MOE_OK)
    return rc;
  return MOE_OK;
}

int launch_pair(const AMaps& ma, const CUtensorMap& mb, const CUtensorMap& mb64, const GemmArgs& g,
                int sm_count, cudaStream_t st) {
  constexpr size_t smem = sizeof(PairStorage) + 1024;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  static std::mutex mu;
  static int clusters_of[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return MOE_ERR_CUDA;
  auto kern = (g.mode == kDgradDH || g.mode == kDgradDX) ? k_grouped_gemm_pair<kPairDgrad>
               : g.gu_out                                  ? k_grouped_gemm_pair<kPairFwdKeep>
                                                           : k_grouped_gemm_pair<kPairFwd>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (clusters_of[dev] == 0) {
      cfg.gridDim = dim3(sm_count & ~1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      clusters_of[dev] = n;
    }
    nclusters = clusters_of[dev];
  }
  if (nclusters > sm_count / 2) nclusters = sm_count / 2;
  GemmArgs ga = g;
  ga.interleave = tuning(MOE_TUNE_PAIR_INTERLEAVE) != 0 ? 1 : 0;
  ga.a_trim = tuning(MOE_TUNE_PAIR_A_TRIM) != 0 ? 1 : 0;
  ga.swap_ab = (g.mode != kDgradDH && g.mode != kDgradDX && tuning(MOE_TUNE_PAIR_SWAP_AB) != 0)
                   ? 1 : 0;
  ga.stream_hint = tuning(MOE_TUNE_PAIR_STREAM_HINT) != 0 ? 1 : 0;
  ga.prefetch = (int)tuning(MOE_TUNE_PAIR_PREFETCH);
  if (launch_kernel(kern, 2 * nclusters, kThreads, smem, st, 2, ma.m128, ma.m64, ma.m32, ma.m16,
                    ma.m8, mb, mb64, ga) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  count_launch();
  return MOE_OK;
}

// The CTA-pair kernel pays off once groups are tall (256-row tiles); small batches keep
// the one-CTA kernel. MOE_TUNE_GEMM_PAIR forces either, MOE_TUNE_PAIR_HALF = 0 runs every
// pair tile as M = 256 (for measurements).
int pair_half_tiles() { return tuning(MOE_TUNE_PAIR_HALF) != 0 ? 1 : 0; }

// M tiles per band of the CTA-pair tile order (see decode_pair_tile); 0 picks the default.
int band_of(int knob) {
  const int v = (int)tuning(knob);
  return v > 0 ? v : 1;
}

bool use_pair_kernel(int T) {
  const int64_t v = tuning(MOE_TUNE_GEMM_PAIR);
  if (v == 0) return false;
  if (v == 1) return true;
  return T >= 1024;
}

// W_r fp32 [E, H] -> bf16 [E, 3H] = [hi | mid | lo] with hi + mid + lo == w exactly:
// hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid); each difference is exact in
// fp32 (the significands shrink by 8 bits per step), and so is every product x * part
// for bf16 x, so the three-part GEMM forms the same products as the fp32 one.
__global__ void __launch_bounds__(256) k_split_router_weight(const float4* __restrict__ w,
                                                             __nv_bfloat16* __restrict__ out,
                                                             int E, int H) {
  pdl_launch_dependents();
  pdl_wait();
  const int H4 = H / 4;                       // four weights per thread step
  const size_t n = (size_t)E * H4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = i / H4, k = (i - e * H4) * 4;
    const float4 v4 = w[i];
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float hi[4], mid[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      hi[j] = __bfloat162float(__float2bfloat16_rn(v[j]));
      const float r1 = __fsub_rn(v[j], hi[j]);
      mid[j] = __bfloat162float(__float2bfloat16_rn(r1));
      lo[j] = __fsub_rn(r1, mid[j]);             // exact in bf16: at most 8 significant bits
    }
    __nv_bfloat16* row = out + e * 3 * (size_t)H + k;
    *reinterpret_cast<uint2*>(row) = make_uint2(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]));
    *reinterpret_cast<uint2*>(row + H) =
        make_uint2(pack_bf16x2(mid[0], mid[1]), pack_bf16x2(mid[2], mid[3]));
    *reinterpret_cast<uint2*>(row + 2 * (size_t)H) =
        make_uint2(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]));
  }
}

}  // namespace

// Router logits: 128 x 128 tiles, K = 3H (the three weight parts); the tensor cores
// accumulate kRouterChunk k-blocks at a time and the epilogue sums the chunks in fp32.
constexpr int kRouterChunk = 6;
// k-blocks per split at least (MOE_TUNE_ROUTER_MIN_SPLIT, 12 by default)
int router_min_split() { return (int)tuning(MOE_TUNE_ROUTER_MIN_SPLIT); }

// The router GEMM's N tile: 256 logits when the 256-wide tiles fill a wave of SMs (the
// A tile is then read once per 256 logits), else 128 (twice the tiles for a small batch:
// decode's 128 tokens x 768 logits fill 144 CTAs with the K split instead of 72).
// MOE_TUNE_ROUTER_N = 192 / 256 forces that width where 256-logit tiles fill a wave (for
// measurements).
int router_n_override() { return (int)tuning(MOE_TUNE_ROUTER_N); }

int router_tile_n(int T, int E, int sm_count) {
  const long mt = (T + BM - 1) / BM;
  const long tiles256 = mt * ((E + 255) / 256);
  if (tiles256 < sm_count) return 128;
  if (router_n_override()) return router_n_override();
  // whole waves times the tile width (a tile's time grows with its width): 192-logit
  // tiles when they need less of it, e.g. 8192 tokens x 768 experts on 148 SMs: 256 tiles
  // in two waves of 192 against 192 tiles in two waves of 256
  const long tiles192 = mt * ((E + 191) / 192);
  const long c256 = (tiles256 + sm_count - 1) / sm_count * 256;
  const long c192 = (tiles192 + sm_count - 1) / sm_count * 192;
  return c192 < c256 ? 192 : 256;
}

int router_tc_splitk(int T, int E, int H, int sm_count) {
  if (sm_count > 160) sm_count = 160;
  if (sm_count < 1) sm_count = 1;
  const int nl = router_tile_n(T, E, sm_count);
  const long tiles = (long)((T + BM - 1) / BM) * ((E + nl - 1) / nl);
  const int kblocks = 3 * H / BK;
  if (tiles <= 0) return 1;
  // a full wave already: no partial slices (splitting K to fill the last wave better
  // measured slower at T = 8192: 0.322 vs 0.292 ms for the route call)
  if (tiles >= sm_count) return 1;
  long s = (2L * sm_count + tiles - 1) / tiles;
  long smax = kblocks / router_min_split();
  if (smax > 64) smax = 64;
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  const int kbp = (kblocks + (int)s - 1) / (int)s;      // no empty split
  return (kblocks + kbp - 1) / kbp;
}

size_t router_tc_scratch_bytes(int T, int E, int H) {
  int S = 1;                                          // the most slices any SM count takes
  for (int sm = 1; sm <= 160; ++sm) {
    const int s_sm = router_tc_splitk(T, E, H, sm);
    if (s_sm > S) S = s_sm;
  }
  size_t b = (size_t)E * 3 * H * 2;                  // split weight
  b = (b + 1023) / 1024 * 1024;
  if (S > 1) b += (size_t)S * T * E * sizeof(float); // per-split partial logits
  return b;
}

int launch_router_pack(const float* w_router, void* w_packed, int E, int H, int sm_count,
                       cudaStream_t st) {
  const size_t n = (size_t)E * H / 4;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 8 * sm_count) blocks = 8 * sm_count;
  const cudaError_t e = launch_kernel(k_split_router_weight, blocks, 256, 0, st, 1,
                                      reinterpret_cast<const float4*>(w_router),
                                      static_cast<__nv_bfloat16*>(w_packed), E, H);
  count_launch();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_router_logits_tc(const void* x, const float* w_router, const void* w_packed, int T,
                            int E, int H, float* logits, void* scratch, int sm_count,
                            ZeroSpec zero, cudaStream_t st, const float** src_out,
                            int* splits_out) {
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  __nv_bfloat16* wsplit = static_cast<__nv_bfloat16*>(scratch);
  size_t off = ((size_t)E * 3 * H * 2 + 1023) / 1024 * 1024;
  float* partial = reinterpret_cast<float*>(static_cast<char*>(scratch) + off);
  if (w_packed) {
    wsplit = static_cast<__nv_bfloat16*>(const_cast<void*>(w_packed));
  } else {
    const size_t n = (size_t)E * H / 4;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 8 * sm_count) blocks = 8 * sm_count;
    const cudaError_t e = launch_kernel(k_split_router_weight, blocks, 256, 0, st, 1,
                                        reinterpret_cast<const float4*>(w_router), wsplit, E, H);
    count_launch();
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  CUtensorMap mx, mw;
  int rc;
  const int nl = router_tile_n(T, E, sm_count > 160 ? 160 : sm_count);
  if ((rc = make_map(&mx, x, (uint64_t)T, H)) != MOE_OK) return rc;
  // B boxes: 128 rows (two per 256-logit tile) or one 192-row box
  if ((rc = make_map(&mw, wsplit, (uint64_t)E, 3ull * H, nl == 192 ? 192 : BM)) != MOE_OK)
    return rc;
  const int S = router_tc_splitk(T, E, H, sm_count);
  GemmArgs g{};
  g.mode = kLogits;
  g.n_ffn = 1;
  g.dense_rows = T;
  g.kblocks = 3 * H / BK;
  g.a_kwrap = H / BK;
  g.ksplit = S;
  g.kb_per_split = (g.kblocks + S - 1) / S;
  g.kchunk = kRouterChunk;
  g.logit_n = nl;
  g.n_tiles = (E + g.logit_n - 1) / g.logit_n;
  g.b_rows = 0;
  g.b_second = BM;
  g.n_valid = E;
  g.ld_out = E;
  g.out = S > 1 ? static_cast<void*>(partial) : static_cast<void*>(logits);
  g.split_stride = (long long)T * E;
  g.zero = zero;
  if ((rc = launch_one(mx, mw, g, sm_count, st)) != MOE_OK) return rc;
  // with S > 1 the top-K kernel sums the partial slices in split order
  *src_out = S > 1 ? partial : logits;
  *splits_out = S;
  return MOE_OK;
}

int launch_grouped_ffn_tc(const void* x, const void* x_perm, const int32_t* offsets,
                          const void* w_gate_up,
                          const void* w_down, const int32_t* perm_token, const float* row_gate,
                          void* h, void* y_perm, float* out_acc, void* gu_out, int T, int H,
                          int I, int n_ffn, int K, float scale, int fused, int* status,
                          int sm_count, cudaStream_t st) {
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  const uint64_t rows = (uint64_t)T * K + BM;   // x_perm / h / y_perm allocation rows
  CUtensorMap mx, mwgu, mwgu64, mh, mwd;
  AMaps ax, ah;
  int rc;
  // A of the gate/up GEMM: the permuted rows, or the token rows gathered through perm_token
  if (x_perm) {
    if ((rc = make_map(&mx, x_perm, rows, H)) != MOE_OK) return rc;
  } else {
    if ((rc = make_map(&mx, x, (uint64_t)T, H, 1)) != MOE_OK) return rc;
  }
  const bool pair = use_pair_kernel(T) && x_perm != nullptr;
  if ((rc = make_map(&mwgu, w_gate_up, (uint64_t)n_ffn * 2 * I, H)) != MOE_OK) return rc;
  if (pair && (rc = make_map(&mwgu64, w_gate_up, (uint64_t)n_ffn * 2 * I, H, 64)) != MOE_OK)
    return rc;
  if ((rc = make_map(&mh, h, rows, I)) != MOE_OK) return rc;
  if (pair && ((rc = make_amaps(&ax, x_perm, rows, H)) != MOE_OK ||
               (rc = make_amaps(&ah, h, rows, I)) != MOE_OK))
    return rc;
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
  g1.offsets = offsets;
  g1.gather_tok = x_perm ? nullptr : perm_token;
  g1.out = h;
  g1.gu_out = gu_out;
  g1.status = status;
  g1.ksplit = 1;
  g1.kb_per_split = g1.kblocks;
  g1.half_tiles = pair ? pair_half_tiles() : 0;
  g1.band = band_of(MOE_TUNE_GATE_UP_BAND);
  g1.test_stall = take_test_stall() ? 1 : 0;
  // CTA pairs: an expert's whole 256-row tiles on the pair kernel, the rest of its rows
  // (at most 128) on the one-CTA kernel (pair_rows), each GEMM as two launches
  const bool split = pair && tuning(MOE_TUNE_PAIR_TAILS) != 0;
  if (split) {
    g1.row_split = 1;
    if ((rc = launch_pair(ax, mwgu, mwgu64, g1, sm_count, st)) != MOE_OK) return rc;
    GemmArgs t1 = g1;
    t1.row_split = 2;
    t1.half_tiles = 0;
    t1.test_stall = 0;
    if ((rc = launch_one(mx, mwgu, t1, sm_count, st)) != MOE_OK) return rc;
  } else if ((rc = pair ? launch_pair(ax, mwgu, mwgu64, g1, sm_count, st)
                        : launch_one(mx, mwgu, g1, sm_count, st)) != MOE_OK) {
    return rc;
  }

  GemmArgs g2{};
  g2.mode = fused ? kDownAtomic : kDownStore;
  g2.n_ffn = n_ffn;
  g2.kblocks = I / BK;
  g2.n_tiles = (H + 255) / 256;
  g2.b_rows = H;
  g2.b_second = BM;
  g2.n_valid = H;
  g2.ld_out = H;
  g2.offsets = offsets;
  g2.out = fused ? static_cast<void*>(out_acc) : y_perm;
  g2.perm_token = perm_token;
  g2.row_gate = row_gate;
  g2.scale = scale;
  g2.status = status;
  g2.ksplit = 1;
  g2.kb_per_split = g2.kblocks;
  g2.half_tiles = pair ? pair_half_tiles() : 0;
  g2.band = band_of(MOE_TUNE_DOWN_BAND);
  if (split) {
    g2.row_split = 1;
    if ((rc = launch_pair(ah, mwd, mwd, g2, sm_count, st)) != MOE_OK) return rc;
    GemmArgs t2 = g2;
    t2.row_split = 2;
    t2.half_tiles = 0;
    return launch_one(mh, mwd, t2, sm_count, st);
  }
  return pair ? launch_pair(ah, mwd, mwd, g2, sm_count, st)
              : launch_one(mh, mwd, g2, sm_count, st);
}

int launch_gate_up_raw(const void* x_perm, const int32_t* offsets, const void* w_gate_up,
                       void* gu, int T, int H, int I, int n_ffn, int K, int* status, int sm_count,
                       cudaStream_t st) {
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  const uint64_t rows = (uint64_t)T * K + BM;
  const bool pair = use_pair_kernel(T);
  CUtensorMap mx, mwgu, mwgu64;
  AMaps ax;
  int rc;
  if ((rc = make_map(&mx, x_perm, rows, H)) != MOE_OK) return rc;
  if ((rc = make_map(&mwgu, w_gate_up, (uint64_t)n_ffn * 2 * I, H)) != MOE_OK) return rc;
  if (pair && ((rc = make_map(&mwgu64, w_gate_up, (uint64_t)n_ffn * 2 * I, H, 64)) != MOE_OK ||
               (rc = make_amaps(&ax, x_perm, rows, H)) != MOE_OK))
    return rc;
  GemmArgs g{};
  g.mode = kGateUp;
  g.gu_raw = 1;
  g.n_ffn = n_ffn;
  g.kblocks = H / BK;
  g.n_tiles = I / BM;
  g.b_rows = 2 * I;
  g.b_second = I;
  g.n_valid = I;
  g.ld_out = 2 * I;
  g.offsets = offsets;
  g.out = gu;
  g.status = status;
  g.ksplit = 1;
  g.kb_per_split = g.kblocks;
  g.half_tiles = pair ? pair_half_tiles() : 0;
  // the same split as the forward, so that G | U come out with the forward's bits
  if (pair && tuning(MOE_TUNE_PAIR_TAILS) != 0) {
    g.row_split = 1;
    if ((rc = launch_pair(ax, mwgu, mwgu64, g, sm_count, st)) != MOE_OK) return rc;
    g.row_split = 2;
    g.half_tiles = 0;
    return launch_one(mx, mwgu, g, sm_count, st);
  }
  return pair ? launch_pair(ax, mwgu, mwgu64, g, sm_count, st)
              : launch_one(mx, mwgu, g, sm_count, st);
}

// MOE_TUNE_BWD_PAIR = 0 keeps the dgrad GEMMs on the one-CTA backward kernel (for
// measurements).
bool dgrad_use_pair(int T) {
  if (tuning(MOE_TUNE_BWD_PAIR) == 0) return false;
  return use_pair_kernel(T);
}

int launch_dgrad_pair(int mode_dx, const void* a_rows, int a_cols, const void* w, int b_rows,
                      int n, const void* gu, void* out, const int32_t* offsets, int T, int K,
                      int n_ffn, int* status, int sm_count, cudaStream_t st) {
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  const uint64_t rows = (uint64_t)T * K + BM;   // row buffers' allocation rows
  AMaps ma;
  CUtensorMap mb;
  int rc;
  if ((rc = make_amaps(&ma, a_rows, rows, (uint64_t)a_cols)) != MOE_OK) return rc;
  if ((rc = make_map(&mb, w, (uint64_t)n_ffn * b_rows, (uint64_t)n, 64)) != MOE_OK) return rc;
  GemmArgs g{};
  g.mode = mode_dx ? kDgradDX : kDgradDH;
  g.n_ffn = n_ffn;
  g.kblocks = a_cols / BK;
  g.n_tiles = (n + BN - 1) / BN;
  g.b_rows = b_rows;
  g.n_valid = n;
  g.ld_out = mode_dx ? n : 2 * n;
  g.offsets = offsets;
  g.out = out;
  g.gu_in = static_cast<const __nv_bfloat16*>(gu);
  g.status = status;
  g.ksplit = 1;
  g.kb_per_split = g.kblocks;
  g.half_tiles = pair_half_tiles();
  return launch_pair(ma, mb, mb, g, sm_count, st);
}

int make_tma_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
  if (get_encoder() != MOE_OK) return MOE_ERR_CUDA;
  return make_map(m, base, rows, cols, box_rows);
}

}  // namespace moe
