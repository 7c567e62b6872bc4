// Host-side launchers of the M²RNN kernels (internal to libm2rnn.so).
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"

namespace m2rnn {

// Forward scan of the bf16 modes.  K, V in {16, 32, 64, 128}.  Few pairs of
// 64-column states run the row kernel (fwd_rows.cu, one warp per state row);
// otherwise the tcgen05 kernel, which with few (b, h) pairs splits the rows
// over several CTAs per pair.  Either way fwd_tc_slices(...) CTAs serve a pair
// and the slices' partial readouts (p.ypart) are summed into y.
cudaError_t launch_fwd_tc(const Params& p, cudaStream_t s);
// Row kernel (V = 64, at most 148 CTAs of 8 rows); fwd_rows_per_cta gives its
// rows per CTA, or 0 when it does not take the problem.
cudaError_t launch_fwd_rows(const Params& p, cudaStream_t s);
int fwd_rows_per_cta(int B, int H, int K, int V);
// y = the sum of p.slices partial readouts p.ypart, in slice order.
cudaError_t launch_y_reduce(const Params& p, cudaStream_t s);
// Register-resident mma.sync forward (V = 64, K in {16, 32, 64}).
cudaError_t launch_fwd_mma(const Params& p, cudaStream_t s);
bool fwd_mma_supported(int K, int V);
// fp32 CUDA-core forward (debug mode).
cudaError_t launch_fwd_fp32(const Params& p, cudaStream_t s);
// fp32 CUDA-core backward (debug mode): chunked recompute + BPTT + dW reduce.
cudaError_t launch_bwd_fp32(const Params& p, cudaStream_t s);
// tcgen05 backward (bf16 inputs): chunked recompute + BPTT + dW reduce.
cudaError_t launch_bwd_tc(const Params& p, cudaStream_t s);
// Deterministic dW[h] = sum over b and slices of dW_part[b, h, slice] (fixed ascending order).
cudaError_t launch_dw_reduce(const Params& p, cudaStream_t s);
// Grouped k / q: dk, dq [B, G, T, K] = sums over each group's heads of the
// per-head dk_part, dq_part [B, H, T, K] (ascending head order).
cudaError_t launch_qk_group_reduce(const Params& p, const float* dk_part, const float* dq_part, float* dk, float* dq,
                                   cudaStream_t s);

// Shapes the tensor-core backward supports: K, V in {16, 32, 64, 128} and
// checkpoint stride <= 16 (V = 64 with K >= 32 in bwd_tc.cu, the rest in the
// general-shape kernel of bwd_tcg.cu).
bool bwd_tc_supported(int K, int V, int C);
// General-shape tensor-core backward (bwd_tcg.cu).
bool bwd_tcg_supported(int K, int V, int C);
int bwd_tcg_slices(int K, int V);
size_t bwd_tcg_workspace(int B, int H, int T, int K, int V, int C);
cudaError_t launch_bwd_tcg(const Params& p, cudaStream_t s);
// Row slices (CTAs per (b, h)) of the bf16 forward.
int fwd_tc_slices(int B, int H, int K, int V);
// SMs of a B200 (the only target); used to decide when rows are sliced.
constexpr int kNumSMs = 148;
// Row slices (CTAs per (b, h)) of the tensor-core backward for a K x V state
// and checkpoint stride C.
int bwd_tc_slices(int K, int V, int C);

// Workspace bytes beyond the 256-byte status header.
size_t bwd_fp32_workspace(int B, int H, int K, int V, int C);
size_t bwd_tc_workspace(int B, int H, int T, int K, int V, int C);

}  // namespace m2rnn
