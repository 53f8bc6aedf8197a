// route.cu -- entmax block routing over chunk summaries (MiniCPM-4-8B-NSA page, DashAttention,
// "How it works", stage 2): every query row scores the chunk summaries it may see,
// s_c = scaling_factor * q . sigma_c / sqrt(d), and routes by alpha-entmax over those scores,
// pi = [(alpha - 1) s - tau]_+^(1/(alpha - 1)) with sum(pi) = 1, by the bracketed Halley +
// bisection search of the attention kernels (Search in common.cuh).  The rows see the chunks
// before their own and, with estimate_diagonal, their own (causal), or every chunk.
// One warp per query row.  Lane l owns the chunks l, l + 32, ...: it writes their z = (alpha - 1) s
// into the row of pi, reads them back at every search step and finally overwrites them with p, so
// no lane ever reads an element another lane writes.  With scores_ready the rows of pi already
// hold z for every chunk (route_scores_kernel, tensor cores), and the warp only searches.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace ea {
namespace {

constexpr int kRouteRowsPerCta = 8;

template <typename T, int BK>
__global__ void __launch_bounds__(32 * kRouteRowsPerCta)
    route_chunks_kernel(const T* __restrict__ q, const T* __restrict__ sig, float* __restrict__ pi,
                        float* __restrict__ tau, int B, int Hq, int Hkv, int T_, int d, int nc,
                        int chunk, float alpha, float beta, float zscale, int n_iter, int causal,
                        int diag, int scores_ready) {
  // grid: (row blocks of one (batch, head), heads, batches) -- no index divisions
  const int i = blockIdx.x * kRouteRowsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= T_) return;  // whole warps leave together
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t row = (static_cast<int64_t>(b) * Hq + h) * T_ + i;
  const int hk = h / (Hq / Hkv);
  int n = nc;
  if (causal) n = min(nc, i / chunk + (diag ? 1 : 0));
  float* pr = pi + row * nc;
  const T* qr = q + row * d;
  const T* sg = sig + (static_cast<int64_t>(b) * Hkv + hk) * nc * d;
  for (int c = n + lane; c < nc; c += 32) pr[c] = 0.f;  // chunks the row may not see
  if (n == 0) {
    if (lane == 0 && tau) tau[row] = INFINITY;
    return;
  }
  const unsigned full = 0xffffffffu;
  float m = -INFINITY;
  for (int c = lane; c < n; c += 32) {
    float z;
    if (scores_ready) {
      z = pr[c];
    } else {
      const T* sc = sg + static_cast<int64_t>(c) * d;
      float acc = 0.f;
      for (int e = 0; e < d; ++e) acc = fmaf(load_elem(qr, e), load_elem(sc, e), acc);
      z = zscale * acc;
      pr[c] = z;
    }
    m = fmaxf(m, z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(full, m, o));
  Search sr;
  sr.init(m, n, alpha);
  for (int it = 0; it < n_iter; ++it) {
    const float t = sr.tau;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f;
    for (int c = lane; c < n; c += 32) {
      const float y = pr[c] - t;
      if (y > 0.f) {
        float a0, a1, a2;
        entmax_powers<BK>(y, beta, a0, a1, a2);
        s0 += a0;
        s1 += a1;
        s2 += a2;
      }
    }
    // butterfly sums: identical bits in every lane, so the step and the exit are uniform
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s0 += __shfl_xor_sync(full, s0, o);
      s1 += __shfl_xor_sync(full, s1, o);
      s2 += __shfl_xor_sync(full, s2, o);
    }
    sr.step<BK>(s0, s1, s2, beta);
    if (sr.settled()) break;
  }
  const float t = sr.tau;
  for (int c = lane; c < n; c += 32) pr[c] = entmax_p<BK>(pr[c] - t, beta);
  if (tau && lane == 0) tau[row] = t;
}

template <typename T>
cudaError_t launch_route_t(const void* q, const void* sig, float* pi, float* tau, int B, int Hq,
                           int Hkv, int T_, int d, int nc, int chunk, float alpha, int n_iter,
                           int causal, int diag, float scaling, int scores_ready,
                           cudaStream_t s) {
  const float beta = 1.f / (alpha - 1.f);
  const float zscale = (alpha - 1.f) * scaling / sqrtf(static_cast<float>(d));
  const dim3 grid(static_cast<unsigned>((T_ + kRouteRowsPerCta - 1) / kRouteRowsPerCta),
                  static_cast<unsigned>(Hq), static_cast<unsigned>(B));
  const dim3 block(32 * kRouteRowsPerCta);
  const T* qp = static_cast<const T*>(q);
  const T* sp = static_cast<const T*>(sig);
#define EA_ROUTE_LAUNCH(BKV)                                                                   \
  route_chunks_kernel<T, BKV><<<grid, block, 0, s>>>(qp, sp, pi, tau, B, Hq, Hkv, T_, d, nc,   \
                                                     chunk, alpha, beta, zscale, n_iter,       \
                                                     causal, diag, scores_ready)
  switch (beta_kind(beta)) {
    case kBetaOne: EA_ROUTE_LAUNCH(kBetaOne); break;
    case kBetaTwo: EA_ROUTE_LAUNCH(kBetaTwo); break;
    case kBetaNear3: EA_ROUTE_LAUNCH(kBetaNear3); break;
    default: EA_ROUTE_LAUNCH(kBetaGeneral);
  }
#undef EA_ROUTE_LAUNCH
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_chunks(const void* q, const void* sig, float* pi, float* tau, int B,
                                int Hq, int Hkv, int T, int d, int nc, int chunk, float alpha,
                                int n_iter, int causal, int diag, float scaling, int dtype,
                                int scores_ready, cudaStream_t s) {
  return dtype == 0 ? launch_route_t<float>(q, sig, pi, tau, B, Hq, Hkv, T, d, nc, chunk, alpha,
                                            n_iter, causal, diag, scaling, scores_ready, s)
                    : launch_route_t<__nv_bfloat16>(q, sig, pi, tau, B, Hq, Hkv, T, d, nc, chunk,
                                                    alpha, n_iter, causal, diag, scaling,
                                                    scores_ready, s);
}

}  // namespace ea
