// rows.cu -- standalone row-wise alpha-entmax (AdaSplash page, "Triton Entmax (Optimized Entmax
// Activation)"): for every row x of a matrix, p = [(alpha - 1) x - tau]_+^(1/(alpha - 1)) with
// tau such that sum(p) = 1, found by the same bracketed Halley + bisection search as the
// attention kernels' tau pass (Search in common.cuh), stopping early once tau has settled.
// One warp per row.  The search steps sum over the row's window (the keys that can carry p > 0),
// gathered once into shared memory; a row whose window does not fit re-reads the row from global
// memory (L1) at every step, so any row length works.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace ea {
namespace {

constexpr int kRowsPerCta = 8;
constexpr int kRowWin = 1024;  // window scores a warp keeps in shared memory

template <typename T, int BK>
__global__ void __launch_bounds__(32 * kRowsPerCta)
    entmax_rows_kernel(const T* __restrict__ x, int64_t ldx, T* __restrict__ p, int64_t ldp,
                       float* __restrict__ tau, int rows, int n, float alpha, float beta,
                       int n_iter) {
  const int row = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;  // whole warps leave together
  const T* xr = x + row * ldx;
  T* pr = p + row * ldp;
  const float am1 = alpha - 1.f;
  const unsigned full = 0xffffffffu;
  float m = -INFINITY;
  for (int j = lane; j < n; j += 32) m = fmaxf(m, load_elem(xr, j));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(full, m, o));
  Search sr;
  sr.init(am1 * m, n, alpha);
  // Every key with p > 0 has z = (alpha - 1) x > tau >= m_z - 1, the lower end of the bracket,
  // which tau never leaves; so the warp gathers the z of that window (widened by a rounding
  // margin: keys below tau add nothing to any step) into a shared-memory list, and the steps sum
  // over the list instead of sweeping the whole row each time.  A row with more than kRowWin keys
  // in the window sweeps the row at every step.
  __shared__ float win_all[kRowsPerCta][kRowWin];
  float* win = win_all[threadIdx.x >> 5];
  {
    const float floor_z = sr.lo - 1e-3f * (fabsf(sr.lo) + 1.f);
    const unsigned below = (1u << lane) - 1u;
    int w = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const float z = j < n ? am1 * load_elem(xr, j) : -INFINITY;
      const bool in = z > floor_z;
      const unsigned bal = __ballot_sync(full, in);
      const int at = w + __popc(bal & below);
      if (in && at < kRowWin) win[at] = z;
      w += __popc(bal);
    }
    if (w <= kRowWin) {
      __syncwarp();  // the list is visible to every lane of the warp
      for (int it = 0; it < n_iter; ++it) {
        const float t = sr.tau;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
        for (int e = lane; e < w; e += 32) {
          const float y = win[e] - t;
          if (y > 0.f) {
            float a, b, c;
            entmax_powers<BK>(y, beta, a, b, c);
            s0 += a;
            s1 += b;
            s2 += c;
          }
        }
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
      for (int j = lane; j < n; j += 32)
        store_elem(pr, j, entmax_p<BK>(am1 * load_elem(xr, j) - t, beta));
      if (tau && lane == 0) tau[row] = t;
      return;
    }
  }
  for (int it = 0; it < n_iter; ++it) {
    const float t = sr.tau;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f;
    for (int j = lane; j < n; j += 32) {
      const float y = am1 * load_elem(xr, j) - t;
      if (y > 0.f) {
        float a, b, c;
        entmax_powers<BK>(y, beta, a, b, c);
        s0 += a;
        s1 += b;
        s2 += c;
      }
    }
    // butterfly sums: every lane ends with the same bits (fp32 addition commutes), so every
    // lane takes the same step and the loop exit below is uniform
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
  for (int j = lane; j < n; j += 32)
    store_elem(pr, j, entmax_p<BK>(am1 * load_elem(xr, j) - t, beta));
  if (tau && lane == 0) tau[row] = t;
}

template <typename T>
cudaError_t launch_rows_t(const void* x, int64_t ldx, void* p, int64_t ldp, float* tau, int rows,
                          int n, float alpha, int n_iter, cudaStream_t s) {
  const float beta = 1.f / (alpha - 1.f);
  const dim3 grid((rows + kRowsPerCta - 1) / kRowsPerCta);
  const dim3 block(32 * kRowsPerCta);
  const T* xp = static_cast<const T*>(x);
  T* pp = static_cast<T*>(p);
  switch (beta_kind(beta)) {
    case kBetaOne:
      entmax_rows_kernel<T, kBetaOne><<<grid, block, 0, s>>>(xp, ldx, pp, ldp, tau, rows, n,
                                                             alpha, beta, n_iter);
      break;
    case kBetaTwo:
      entmax_rows_kernel<T, kBetaTwo><<<grid, block, 0, s>>>(xp, ldx, pp, ldp, tau, rows, n,
                                                             alpha, beta, n_iter);
      break;
    case kBetaNear3:
      entmax_rows_kernel<T, kBetaNear3><<<grid, block, 0, s>>>(xp, ldx, pp, ldp, tau, rows,
                                                                 n, alpha, beta, n_iter);
      break;
    default:
      entmax_rows_kernel<T, kBetaGeneral><<<grid, block, 0, s>>>(xp, ldx, pp, ldp, tau, rows,
                                                                 n, alpha, beta, n_iter);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_entmax_rows(const void* x, int64_t ldx, void* p, int64_t ldp, float* tau,
                               int rows, int n, float alpha, int n_iter, int dtype,
                               cudaStream_t s) {
  return dtype == 0
             ? launch_rows_t<float>(x, ldx, p, ldp, tau, rows, n, alpha, n_iter, s)
             : launch_rows_t<__nv_bfloat16>(x, ldx, p, ldp, tau, rows, n, alpha, n_iter, s);
}

}  // namespace ea
