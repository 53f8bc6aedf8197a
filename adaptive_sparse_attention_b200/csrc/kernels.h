// kernels.h -- host-side launchers of the entmax attention kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <cmath>

#include "common.cuh"

namespace ea {

// dtype: 0 = fp32, 1 = bf16.  Each returns cudaSuccess or the launch error.
cudaError_t launch_tau_simt(const Problem& P, int dtype, cudaStream_t s);
cudaError_t launch_tau_fallback(const Problem& P, int dtype, int num_ctas, cudaStream_t s);
cudaError_t launch_out_simt(const Problem& P, int dtype, cudaStream_t s);

// Tensor-core (tcgen05) kernels, bf16 only, d in {64, 128}.
cudaError_t launch_tau_tc(const Problem& P, cudaStream_t s);
// Multi-sweep tau search on the tensor cores for the overflow queue (one CTA per SM at most).
cudaError_t launch_tau_tc_fallback(const Problem& P, int num_ctas, cudaStream_t s);
cudaError_t launch_out_tc(const Problem& P, cudaStream_t s);
// Output of the query tiles that are not pending, from the support lists the tau pass recorded
// (bf16 values, d in {64, 128}).
cudaError_t launch_out_support(const Problem& P, cudaStream_t s);
// Warm-up keys of the tensor-core tau pass (P.norms, P.warm); nothing when P.warm_levels == 0.
cudaError_t launch_warm(const Problem& P, cudaStream_t s);

// Backward pass on the CUDA cores: delta (fp32 per query row), then dq (fp32, written) and dk,
// dv (fp32, accumulated: zero them first).  g is the upstream gradient in the input dtype.
cudaError_t launch_bwd(const Problem& P, int dtype, const void* g, float* delta, float* dq,
                       float* dk, float* dv, cudaStream_t s);

// FP8 screen of the tau pass (screen.cu, bf16, d = 128): e4m3 copies of q (per row) and k (per
// 128-key tile) with their scales and error norms, then per query tile the ascending list of key
// tiles the bf16 tau pass must visit and its count.  q8 [q rows][128] bytes, qst float4 [q rows],
// k8 [kv rows][128] bytes, kst float4 [(B or 1) Hkv slots], list [tiles][nkt_max], count [tiles].
cudaError_t launch_screen(const Problem& P, void* q8, void* qst, void* k8, void* kst, int* list,
                          int* count, cudaStream_t s);

// Entmax block routing over chunk summaries (pi fp32 [B, Hq, T, nc], tau fp32 [B, Hq, T]);
// with scores_ready the rows of pi already hold z = (alpha - 1) scaling q . sigma / sqrt(d).
cudaError_t launch_route_chunks(const void* q, const void* sig, float* pi, float* tau, int B,
                                int Hq, int Hkv, int T, int d, int nc, int chunk, float alpha,
                                int n_iter, int causal, int diag, float scaling, int dtype,
                                int scores_ready, cudaStream_t s);
// z = zscale q . sigma for every (query row, chunk) into z [B, Hq, T, nc] on the tensor cores
// (bf16, d in {64, 128}, q and sig 16-byte aligned); status: the device status word.
cudaError_t launch_route_scores_tc(const void* q, const void* sig, float* z, int B, int Hq,
                                   int Hkv, int T, int d, int nc, float zscale, int* status,
                                   cudaStream_t s);

// Row-wise alpha-entmax of a [rows, n] matrix x (row stride ldx elements) into p (row stride
// ldp); dtype 0 = fp32, 1 = bf16 for both x and p; tau may be null.
cudaError_t launch_entmax_rows(const void* x, int64_t ldx, void* p, int64_t ldp, float* tau,
                               int rows, int n, float alpha, int n_iter, int dtype,
                               cudaStream_t s);

// Records e as the string entmax_attn_last_cuda_error reports and returns ENTMAX_ATTN_ECUDA.
int record_cuda_error(cudaError_t e);

inline int beta_kind(float beta) {
  if (beta == 1.f) return kBetaOne;
  if (beta == 2.f) return kBetaTwo;
  if (fabsf(beta - 3.f) <= kNearIntFrac) return kBetaNear3;
  return kBetaGeneral;
}

}  // namespace ea
