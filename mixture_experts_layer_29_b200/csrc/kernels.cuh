// kernels.cuh - host-side launchers of the layer's kernels (internal to the library).
//
// Every kernel behind these launchers keeps the launch contract of launch.cuh, and one
// more rule: only weights are read through `const __restrict__` pointers, and nothing
// through __ldg. Both compile to non-coherent loads. Those assume the memory stays
// unchanged for the kernel's whole life, and the compiler may schedule them ahead of
// pdl_wait(). A kernel launched as a programmatic dependent is resident while its
// predecessors still write its inputs, and the caller's x may be this library's own
// output from the previous call. So activations are read with plain loads after the wait.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// One launch of one of this library's kernels (counted for moe_launch_count).
void count_launch(int n = 1);

// Current value of a moe_set_tuning switch (MOE_TUNE_*).
int64_t tuning(int knob);
// Reads and clears MOE_TUNE_TEST_STALL: true once per arming.
bool take_test_stall();

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
};
// Cached per device; returns MOE_OK, MOE_ERR_CUDA or MOE_ERR_NO_DEVICE.
int current_device_info(DeviceInfo* info);

// Two int32 buffers that a kernel clears (after its dependency wait) for the kernels
// after it: the router kernels clear the expert counts and the FFN-pick histogram that
// the top-K kernel then accumulates into.
struct ZeroSpec {
  int32_t* a = nullptr;
  int na = 0;
  int32_t* b = nullptr;
  int nb = 0;
#ifdef __CUDACC__
  __device__ __forceinline__ void run(int block, int nblocks, int tid, int nthreads) const {
    const int stride = nblocks * nthreads;
    for (int i = block * nthreads + tid; i < na; i += stride) a[i] = 0;
    for (int i = block * nthreads + tid; i < nb; i += stride) b[i] = 0;
  }
#endif
};

// ---- router -----------------------------------------------------------------------------
// Split-K factor of the logits GEMM for this shape (1 = no partial buffer).
int router_splitk(int T, int E, int H, int sm_count);
size_t router_partial_bytes(int T, int E, int H, int sm_count_max);
cudaError_t launch_router_logits(const void* x, int x_is_bf16, const float* w_router, int T,
                                 int E, int H, float* logits, float* partial, int splitk,
                                 ZeroSpec zero, cudaStream_t st);
cudaError_t launch_splitk_sum(const float* partial, int S, size_t n, float* out, cudaStream_t st);
// bf16 x: logits on the tensor cores with W_r split into three exact bf16 parts.
int router_tc_splitk(int T, int E, int H, int sm_count);
size_t router_tc_scratch_bytes(int T, int E, int H);
// Writes the logits (S == 1) or S partial slices; *src_out / *splits_out tell the top-K
// kernel where to read them.
// w_packed (bf16 [E, 3H] from launch_router_pack) or nullptr: split w_router here.
int launch_router_logits_tc(const void* x, const float* w_router, const void* w_packed, int T,
                            int E, int H, float* logits, void* scratch, int sm_count,
                            ZeroSpec zero, cudaStream_t st, const float** src_out,
                            int* splits_out);
int launch_router_pack(const float* w_router, void* w_packed, int E, int H, int sm_count,
                       cudaStream_t st);
// Softmax / top-K / histograms from S logit slices of T x E (summed in order; S > 1 also
// writes the sum to logits_out).
// counts [E] and nffn_hist [K + 1] must be zero when it runs (a router kernel's ZeroSpec,
// or launch_zero_counts).
cudaError_t launch_route_topk(const float* src, int S, float* logits_out, const float* bias,
                              int T, int E, int n_ffn, int K, int32_t* topk_idx,
                              float* topk_gate, int32_t* counts, int32_t* nffn_hist,
                              float* zgate, int sm_count, cudaStream_t st);
// Whether launch_route_topk reads S slices itself (else sum them first with
// launch_splitk_sum).
bool route_topk_sums_slices(int T, int S, int sm_count);
cudaError_t launch_zero_counts(int32_t* counts, int E, int32_t* nffn_hist, int K, cudaStream_t st);

// rows x cols bf16 row-major tensor map with 128-byte swizzle and a box of 64 columns x
// box_rows rows (no multicast).
int make_tma_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows);

// The backward's dgrad GEMMs on the CTA-pair kernel (B read MN-major), for batches where
// the forward uses it (dgrad_use_pair): mode_dx 0: dh = a_rows . W (W = w_down, b_rows = H,
// n = I) with the SwiGLU backward from gu into out = [dG | dU] (bf16 [rows, 2I]);
// mode_dx 1: dx rows = a_rows . W (a_rows = [dG | dU], W = w_gate_up, b_rows = 2I, n = H)
// into out (fp32 [rows, H]).
bool dgrad_use_pair(int T);
int launch_dgrad_pair(int mode_dx, const void* a_rows, int a_cols, const void* w, int b_rows,
                      int n, const void* gu, void* out, const int32_t* offsets, int T, int K,
                      int n_ffn, int* status, int sm_count, cudaStream_t st);

// ---- backward ------------------------------------------------------------------------------
// The gate/up GEMM again, storing G and U (bf16) instead of h: gu [T*K + 128, 2I].
int launch_gate_up_raw(const void* x_perm, const int32_t* offsets, const void* w_gate_up,
                       void* gu, int T, int H, int I, int n_ffn, int K, int* status, int sm_count,
                       cudaStream_t st);
// dh = dy . W_d[e] with the SwiGLU backward in the epilogue -> dgu [rows, 2I] = [dG | dU];
// dx_perm = dgu . W_gu[e] (fp32); per touched expert d_down[e] = dy^T h and
// d_gate_up[e] = dgu^T x_perm (fp32, experts without rows untouched).
int launch_bwd_gemms(const void* dy, const void* gu, const void* h, const void* x_perm,
                     const int32_t* offsets, const void* w_gate_up, const void* w_down,
                     void* dgu, float* dx_perm, float* d_gate_up, float* d_down, int T, int H,
                     int I, int n_ffn, int K, int* status, int sm_count, cudaStream_t st);

cudaError_t launch_bwd_dy_dgate(const void* dout, const void* x, const void* y_perm,
                                const int32_t* topk_idx, const float* topk_gate,
                                const int32_t* row_of, int T, int H, int K, int n_ffn,
                                float scale, void* dy, float* d_gate, cudaStream_t st);
// logit gradient of every token as three exact bf16 parts dl3 [3][Tp][E] (Tp = T rounded
// up to 64, pad rows zero), the offset tables {0, 3Tp, 0, T} and W_r in bf16
cudaError_t launch_bwd_router(const float* logits, const int32_t* topk_idx, const float* d_gate,
                              int T, int Tp, int E, int K, void* dl3, int32_t* offs,
                              const float* w_router, void* wr16, int H, cudaStream_t st);
// d_router = dL^T x (three parts) and dx = dL_hi W_r (bf16) on the tensor cores
int launch_bwd_router_gemms(const void* dl3, int Tp, const void* x, const void* wr16,
                            const int32_t* offs_k, const int32_t* offs_m, int T, int E, int H,
                            float* d_router, float* dx, int* status, int sm_count,
                            cudaStream_t st);
cudaError_t launch_bwd_dx_combine(const float* dx_perm, const void* dout, const int32_t* topk_idx,
                                  const float* topk_gate, const int32_t* row_of, int T, int H,
                                  int K, int n_ffn, float* dx, cudaStream_t st);

// ---- load-balance loss -------------------------------------------------------------------
size_t lb_partial_bytes(int T, int E);
cudaError_t launch_lb_loss(const float* logits, const int32_t* counts, int T, int E, int n_ffn,
                           int K, double* part, float* prob_mean, float* loss, cudaStream_t st);

// ---- permutation ------------------------------------------------------------------------
cudaError_t launch_permute(const int32_t* topk_idx, const float* topk_gate, const float* zgate,
                           const void* x, int x_is_bf16, int T, int H, int n_ffn, int E, int K,
                           uint32_t* masks, int32_t* crel, int32_t* ecount, int32_t* offsets,
                           int32_t* perm_token, int32_t* row_of, float* row_gate, void* x_perm,
                           float* out_acc, int* status, cudaStream_t st);

// ---- grouped FFN --------------------------------------------------------------------------
// bf16 on tcgen05: gate/up GEMM + SwiGLU -> h, then down GEMM -> y_perm or out_acc.
// x_perm == nullptr: the gate/up GEMM gathers the rows of x through perm_token (TMA gather4).
int launch_grouped_ffn_tc(const void* x, const void* x_perm, const int32_t* offsets,
                          const void* w_gate_up,
                          const void* w_down, const int32_t* perm_token, const float* row_gate,
                          void* h, void* y_perm, float* out_acc, void* gu_out, int T, int H,
                          int I, int n_ffn, int K, float scale, int fused, int* status,
                          int sm_count, cudaStream_t st);
// fp32 on the CUDA cores.
cudaError_t launch_grouped_ffn_simt(const float* x_perm, const int32_t* offsets,
                                    const float* w_gate_up, const float* w_down,
                                    const int32_t* perm_token, const float* row_gate, float* h,
                                    float* y_perm, float* out_acc, int T, int H, int I,
                                    int n_ffn, int K, float scale, int fused, cudaStream_t st);

// ---- combine and PID ----------------------------------------------------------------------
cudaError_t launch_finalize(const float* out_acc, void* out, int out_is_bf16, size_t n,
                            cudaStream_t st);
cudaError_t launch_combine_det(const void* x, const void* y_perm, const float* topk_gate,
                               const int32_t* row_of, const float* zgate, void* out,
                               int is_bf16, int T, int H, int K, float scale, cudaStream_t st);
cudaError_t launch_pid_init(const float* bias, float* pid_state, int n_ffn, cudaStream_t st);
cudaError_t launch_pid_update(const moe_pid_t& pid, const int32_t* counts,
                              const int32_t* nffn_hist, float* bias, float* pid_state,
                              float* stats, int T, int K, int n_ffn, int E, cudaStream_t st);

}  // namespace moe
