// bwd.cu -- backward pass of causal alpha-entmax attention on the CUDA cores (fp32 arithmetic).
//
// Gradients of L = sum(dout * out), from the alpha-entmax Jacobian
//   dp/ds = diag(w) - w w^T / sum(w),   w_j = p_j^(2 - alpha) = [z_j - tau]_+^(beta - 1)
// (Peters, Niculae & Martins 2019, "Sparse Sequence-to-Sequence Models", Proposition 2; the
// AdaSplash page says the forward pass's block mask serves the backward pass too, without a
// formula).  Per query row i, with g_i = dout_i and u_ij = g_i . v_j:
//   delta_i = sum_j w_ij u_ij / sum_j w_ij,   ds_ij = w_ij (u_ij - delta_i)
//   dq_i = sum_j ds_ij k_j / sqrt(d),   dk_j += ds_ij q_i / sqrt(d),   dv_j += p_ij g_i
// p and w come from the forward pass's tau, over the key tiles of the compact lists the tau pass
// wrote (every key with p > 0 lies in a listed tile).
//
//   bwd_delta_kernel  one CTA of 256 threads per query tile, two threads per row r, each owning
//                     half of the head dimension (their partial dot products meet by a shuffle):
//                     sweeps the listed key tiles in chunks of 32 keys and sums w u and w
//                     -> delta.
//   bwd_grad_kernel   the same sweep again: ds and p of each chunk go to shared memory; the two
//                     threads of row r accumulate the two halves of dq_r in registers; then
//                     each thread takes a few keys of the chunk and four of the columns and adds
//                     their dk and dv, summed over the tile's rows, into fp32 global memory with
//                     atomics (several query tiles and the query heads of a group meet on each
//                     key).
//   bwd_support_kernel  with ENTMAX_ATTN_FLAG_SUPPORT, for every query tile whose rows' supports
//                     the forward recorded (bf16): the same gradients over each row's support
//                     list alone -- w, u, delta, ds, dq from the listed keys, dk and dv added
//                     with vector atomics.  The two kernels above then take only the other
//                     (pending) query tiles.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace ea {
namespace {

constexpr int kBT = 256;     // threads per CTA: two per query row
constexpr int kBChunk = 32;  // keys per chunk
constexpr int kXS = kTile + 1;  // padded row of the [key][query row] chunk arrays

template <int D>
struct BwdSmem {
  static constexpr int QS = D + 4;  // padded row of the query and upstream-gradient tiles
  float qs[kTile * QS];
  float gs[kTile * QS];
  float ks[kBChunk * D];
  float vs[kBChunk * D];
  float xs[kBChunk * kXS];  // scores, then ds
  float us[kBChunk * kXS];  // g . v, then p
};

template <typename T, int D>
__device__ __forceinline__ void load_rows(const T* base, int64_t row0, int nrows, float* dst,
                                          int stride, int nrow_tile, int tid) {
  for (int i = tid; i < nrow_tile * D; i += kBT) {
    const int r = i / D, c = i % D;
    dst[r * stride + c] = (r < nrows) ? load_elem(base, (row0 + r) * D + c) : 0.f;
  }
}

// Dot products of row r of rows[128][QS] with the 32 rows of chunk[32][D] -> out[jj][r], by the
// two threads of the row (hf = 0, 1: columns hf D/2 .. hf D/2 + D/2 - 1), whose partial sums
// meet by a shuffle with the neighbouring lane; keys at or past jmax give -inf when masked.
template <int D>
__device__ __forceinline__ void rows_dot_chunk(const float* rows, const float* chunk, float* out,
                                               int r, int hf, int j0, int jmax, bool masked) {
  constexpr int kH4 = D / 8;  // float4 per half row
  const float4* r4 = reinterpret_cast<const float4*>(rows + r * BwdSmem<D>::QS) + hf * kH4;
  const float4* c4 = reinterpret_cast<const float4*>(chunk) + hf * kH4;
  float acc[kBChunk];  // one partial sum per key: each row float4 is loaded once
#pragma unroll
  for (int jj = 0; jj < kBChunk; ++jj) acc[jj] = 0.f;
#pragma unroll 2
  for (int e = 0; e < kH4; ++e) {
    const float4 x = r4[e];
#pragma unroll
    for (int jj = 0; jj < kBChunk; ++jj) {
      const float4 u = c4[jj * (D / 4) + e];
      acc[jj] = fmaf(x.x, u.x, fmaf(x.y, u.y, fmaf(x.z, u.z, fmaf(x.w, u.w, acc[jj]))));
    }
  }
#pragma unroll
  for (int jj = 0; jj < kBChunk; ++jj) {
    const float a = acc[jj] + __shfl_xor_sync(0xffffffffu, acc[jj], 1);
    if (hf == 0) out[jj * kXS + r] = (masked && j0 + jj >= jmax) ? -INFINITY : a;
  }
}

// The listed key tiles of query tile t in chunks of 32 keys: fn(j0) runs after the chunk's keys
// (rows j0 .. j0 + 31 of the sequence, zero past its end) are in ks and its values in vs.
template <typename T, int D, typename Fn>
__device__ __forceinline__ void sweep_listed(const Problem& P, const TileInfo& t,
                                             BwdSmem<D>& sm, int tid, Fn&& fn) {
  const T* kp = static_cast<const T*>(P.k);
  const T* vp = static_cast<const T*>(P.v);
  const int* list = P.list + t.tile_id * P.nkt_max;
  const int cnt = list_count(P, t);
  for (int i = 0; i < cnt; ++i) {
    const int kt = list_tile(P, list, i, t.nkt);
    for (int ch = 0; ch < kTile / kBChunk; ++ch) {
      const int j0 = kt * kTile + ch * kBChunk;
      if (j0 >= t.seq_len) break;
      const int n = min(kBChunk, t.seq_len - j0);
      __syncthreads();  // the previous chunk is no longer read
      load_rows<T, D>(kp, t.khead + t.seq_start + j0, n, sm.ks, D, kBChunk, tid);
      load_rows<T, D>(vp, t.khead + t.seq_start + j0, n, sm.vs, D, kBChunk, tid);
      __syncthreads();
      fn(j0);
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void load_tiles(const Problem& P, const TileInfo& t, const T* g,
                                           BwdSmem<D>& sm, int tid) {
  const int64_t row0 = t.qhead + t.seq_start + t.row0;
  load_rows<T, D>(static_cast<const T*>(P.q), row0, t.nrows, sm.qs, BwdSmem<D>::QS, kTile, tid);
  load_rows<T, D>(g, row0, t.nrows, sm.gs, BwdSmem<D>::QS, kTile, tid);
}

template <typename T, int D, int BK>
__global__ void __launch_bounds__(kBT) bwd_delta_kernel(Problem P, const T* g, float* delta) {
  extern __shared__ __align__(16) unsigned char smem[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem);
  const int tid = threadIdx.x, r = tid >> 1, hf = tid & 1;
  const TileInfo t = map_tile(P, gridDim.x - 1 - blockIdx.x, blockIdx.y, blockIdx.z);
  if (!t.valid) return;
  if (P.from_support && P.pending[t.tile_id] == 0) return;  // bwd_support_kernel's tile
  load_tiles<T, D>(P, t, g, sm, tid);
  const bool row_ok = r < t.nrows;
  const int jmax = row_ok ? (P.causal ? t.row0 + r + 1 : t.seq_len) : 0;
  const int64_t row = t.qhead + t.seq_start + t.row0 + r;
  const float tau = row_ok ? P.tau[row] : INFINITY;
  float a = 0.f, b = 0.f;
  sweep_listed<T, D>(P, t, sm, tid, [&](int j0) {
    rows_dot_chunk<D>(sm.qs, sm.ks, sm.xs, r, hf, j0, jmax, true);
    rows_dot_chunk<D>(sm.gs, sm.vs, sm.us, r, hf, j0, jmax, false);
    __syncwarp();  // both threads of a row see the sums their lane pair wrote
    for (int jj = hf; jj < kBChunk; jj += 2) {  // the two threads split the chunk's keys
      const float x = P.c * sm.xs[jj * kXS + r] - tau;
      if (x > 0.f) {
        float p0, p1, p2;
        entmax_powers<BK>(x, P.beta, p0, p1, p2);
        a = fmaf(p1, sm.us[jj * kXS + r], a);
        b += p1;
      }
    }
  });
  a += __shfl_xor_sync(0xffffffffu, a, 1);
  b += __shfl_xor_sync(0xffffffffu, b, 1);
  if (row_ok && hf == 0) delta[row] = b > 0.f ? a / b : 0.f;
}

template <typename T, int D, int BK>
__global__ void __launch_bounds__(kBT) bwd_grad_kernel(Problem P, const T* g, const float* delta,
                                                       float* dq, float* dk, float* dv) {
  extern __shared__ __align__(16) unsigned char smem[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem);
  constexpr int QS = BwdSmem<D>::QS;
  constexpr int kHalf = D / 2;
  const int tid = threadIdx.x, r = tid >> 1, hf = tid & 1;
  const TileInfo t = map_tile(P, gridDim.x - 1 - blockIdx.x, blockIdx.y, blockIdx.z);
  if (!t.valid) return;
  if (P.from_support && P.pending[t.tile_id] == 0) return;  // bwd_support_kernel's tile
  load_tiles<T, D>(P, t, g, sm, tid);
  const bool row_ok = r < t.nrows;
  const int jmax = row_ok ? (P.causal ? t.row0 + r + 1 : t.seq_len) : 0;
  const int64_t row = t.qhead + t.seq_start + t.row0 + r;
  const float tau = row_ok ? P.tau[row] : INFINITY;
  const float dl = row_ok ? delta[row] : 0.f;
  const float scale = rsqrtf(static_cast<float>(D));
  float acc_q[kHalf];  // columns hf D/2 .. hf D/2 + D/2 - 1 of dq_r
#pragma unroll
  for (int c = 0; c < kHalf; ++c) acc_q[c] = 0.f;
  sweep_listed<T, D>(P, t, sm, tid, [&](int j0) {
    rows_dot_chunk<D>(sm.qs, sm.ks, sm.xs, r, hf, j0, jmax, true);
    rows_dot_chunk<D>(sm.gs, sm.vs, sm.us, r, hf, j0, jmax, false);
    __syncwarp();  // both threads of a row see the sums their lane pair wrote
    for (int jj = 0; jj < kBChunk; ++jj) {
      const float x = P.c * sm.xs[jj * kXS + r] - tau;
      float ds = 0.f, p = 0.f;
      if (x > 0.f) {
        float p0, p1, p2;
        entmax_powers<BK>(x, P.beta, p0, p1, p2);
        ds = p1 * (sm.us[jj * kXS + r] - dl);
        p = p0;
      }
#pragma unroll
      for (int c = 0; c < kHalf; ++c) acc_q[c] = fmaf(ds, sm.ks[jj * D + hf * kHalf + c], acc_q[c]);
      __syncwarp();  // both threads of the row have read the scores of key jj
      if (hf == 0) {
        sm.xs[jj * kXS + r] = ds;
        sm.us[jj * kXS + r] = p;
      }
    }
    __syncthreads();  // every row's ds and p of the chunk are in shared memory
    // dk / dv of the chunk's keys: thread (key group kg, column group cg) sums, over the tile's
    // rows, kKeys keys x 4 columns (columns cg + kCg m, so that a warp's column groups read
    // consecutive words of a query row): 2 kKeys + 8 shared loads per 8 kKeys FMAs
    constexpr int kCg = D / 4;           // column groups
    constexpr int kKeys = kBChunk * kCg / kBT;  // keys per thread
    const int kg = tid / kCg, cg = tid % kCg;
    float ak[kKeys][4], av[kKeys][4];
#pragma unroll
    for (int i = 0; i < kKeys; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        ak[i][m] = 0.f;
        av[i][m] = 0.f;
      }
    for (int rr = 0; rr < kTile; ++rr) {
      float qv[4], gv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        qv[m] = sm.qs[rr * QS + cg + kCg * m];
        gv[m] = sm.gs[rr * QS + cg + kCg * m];
      }
#pragma unroll
      for (int i = 0; i < kKeys; ++i) {
        const float dsr = sm.xs[(kg * kKeys + i) * kXS + rr];
        const float pr = sm.us[(kg * kKeys + i) * kXS + rr];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          ak[i][m] = fmaf(dsr, qv[m], ak[i][m]);
          av[i][m] = fmaf(pr, gv[m], av[i][m]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kKeys; ++i) {
      const int j = j0 + kg * kKeys + i;
      if (j >= t.seq_len) continue;
      const int64_t krow = t.khead + t.seq_start + j;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c = cg + kCg * m;
        if (ak[i][m] != 0.f) atomicAdd(dk + krow * D + c, ak[i][m] * scale);
        if (av[i][m] != 0.f) atomicAdd(dv + krow * D + c, av[i][m]);
      }
    }
  });
  if (row_ok) {
    float* o = dq + row * D + hf * kHalf;
#pragma unroll
    for (int c = 0; c < kHalf; c += 4)
      *reinterpret_cast<float4*>(o + c) =
          make_float4(acc_q[c] * scale, acc_q[c + 1] * scale, acc_q[c + 2] * scale,
                      acc_q[c + 3] * scale);
  }
}

// ------------------------------------------------------------------ backward from the supports --
// w = p^(2 - alpha) (= [z - tau]^(beta - 1)) from the p the forward recorded.
template <int BK>
__device__ __forceinline__ float weight_from_p(float p, float two_minus_alpha) {
  if (BK == kBetaOne) return 1.f;          // alpha = 2
  if (BK == kBetaTwo) return sqrtf(p);     // alpha = 1.5
  return exp2f(two_minus_alpha * __log2f(p));
}

// bf16 row slice of kCols consecutive elements (16-byte aligned) into fp32 registers.
template <int kCols>
__device__ __forceinline__ void load_slice(const __nv_bfloat16* src, float (&x)[kCols]) {
#pragma unroll
  for (int u = 0; u < kCols / 8; ++u) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src) + u);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[h]));
      x[8 * u + 2 * h] = f.x;
      x[8 * u + 2 * h + 1] = f.y;
    }
  }
}

// Sum over the 8 lanes of a row group (lanes 8 m .. 8 m + 7 of the warp).
__device__ __forceinline__ float sum8(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// One CTA of 128 threads per query tile that is not pending; 8 lanes per row, each owning D / 8
// consecutive columns, 16 rows at a time.  First sweep over the row's support list: u = g . v_j
// and w from p -> delta = sum w u / sum w; second sweep: ds = w (u - delta), dq += ds k_j, and
// dk_j += ds q / sqrt(d), dv_j += p g with float4 atomics.  Every lane of a row group runs the
// same trip counts (the shuffles need the whole warp), and list offsets, counts and keys are
// clamped to the tile's list and sequence.
constexpr int kBSupThreads = 128;

template <int D, int BK>
__global__ void __launch_bounds__(kBSupThreads)
    bwd_support_kernel(Problem P, const __nv_bfloat16* g, float* delta, float* dq, float* dk,
                       float* dv) {
  const TileInfo t = map_tile(P, gridDim.x - 1 - blockIdx.x, blockIdx.y, blockIdx.z);
  if (!t.valid || P.pending[t.tile_id] != 0) return;
  constexpr int kCols = D / 8;
  const int l8 = threadIdx.x & 7;
  const float scale = rsqrtf(static_cast<float>(D));
  const float tma = 2.f - P.alpha;
  const int2* list = P.sup + t.tile_id * kSupPerTile;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(P.q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(P.k);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(P.v);
  const int64_t kv0 = t.khead + t.seq_start;  // key row of the sequence's first key
  // row groups of a warp run a common trip count: the warp's largest support
  for (int r0 = 0; r0 < t.nrows; r0 += kBSupThreads / 8) {
    const int r = r0 + (threadIdx.x >> 3);
    const bool ok = r < t.nrows;
    const int64_t row = t.qhead + t.seq_start + t.row0 + (ok ? r : 0);
    const int idx = ok ? P.sup_idx[row] : 0;
    const int first = min(idx & 0xffff, kSupPerTile);
    const int n = ok ? min(max(idx >> 16, 0), kSupPerTile - first) : 0;
    int nmax = n;
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) nmax = max(nmax, __shfl_xor_sync(0xffffffffu, nmax, o));
    float gi[kCols];
    load_slice<kCols>(g + row * D + l8 * kCols, gi);
    float sw = 0.f, swu = 0.f;
    for (int e = 0; e < nmax; ++e) {
      const bool has = e < n;
      const int2 en = has ? list[first + e] : make_int2(0, 0);
      const int j = min(max(en.x, 0), t.seq_len - 1);
      float vj[kCols];
      load_slice<kCols>(vb + (kv0 + j) * D + l8 * kCols, vj);
      float u = 0.f;
#pragma unroll
      for (int c = 0; c < kCols; ++c) u = fmaf(gi[c], vj[c], u);
      u = sum8(u);
      const float p = __int_as_float(en.y);
      const float w = (has && p > 0.f) ? weight_from_p<BK>(p, tma) : 0.f;
      sw += w;
      swu = fmaf(w, u, swu);
    }
    const float dl = sw > 0.f ? swu / sw : 0.f;
    float qi[kCols], aq[kCols];
    load_slice<kCols>(qb + row * D + l8 * kCols, qi);
#pragma unroll
    for (int c = 0; c < kCols; ++c) aq[c] = 0.f;
    for (int e = 0; e < nmax; ++e) {
      const bool has = e < n;
      const int2 en = has ? list[first + e] : make_int2(0, 0);
      const int j = min(max(en.x, 0), t.seq_len - 1);
      float vj[kCols], kj[kCols];
      load_slice<kCols>(vb + (kv0 + j) * D + l8 * kCols, vj);
      load_slice<kCols>(kb + (kv0 + j) * D + l8 * kCols, kj);
      float u = 0.f;
#pragma unroll
      for (int c = 0; c < kCols; ++c) u = fmaf(gi[c], vj[c], u);
      u = sum8(u);
      if (!has) continue;  // the shuffles are done; the rest is this row group's own
      const float p = __int_as_float(en.y);
      const float w = p > 0.f ? weight_from_p<BK>(p, tma) : 0.f;
      const float ds = w * (u - dl);
#pragma unroll
      for (int c = 0; c < kCols; ++c) aq[c] = fmaf(ds, kj[c], aq[c]);
      float4* dkr = reinterpret_cast<float4*>(dk + (kv0 + j) * D + l8 * kCols);
      float4* dvr = reinterpret_cast<float4*>(dv + (kv0 + j) * D + l8 * kCols);
      const float dss = ds * scale;
#pragma unroll
      for (int c = 0; c < kCols; c += 4) {
        atomicAdd(dkr + c / 4, make_float4(dss * qi[c], dss * qi[c + 1], dss * qi[c + 2],
                                           dss * qi[c + 3]));
        atomicAdd(dvr + c / 4, make_float4(p * gi[c], p * gi[c + 1], p * gi[c + 2],
                                           p * gi[c + 3]));
      }
    }
    if (!ok) continue;
    float4* dqr = reinterpret_cast<float4*>(dq + row * D + l8 * kCols);
#pragma unroll
    for (int c = 0; c < kCols; c += 4)
      dqr[c / 4] = make_float4(aq[c] * scale, aq[c + 1] * scale, aq[c + 2] * scale,
                               aq[c + 3] * scale);
    if (l8 == 0) delta[row] = dl;
  }
}

template <int D>
cudaError_t launch_bwd_support_d(const Problem& P, const void* g, float* delta, float* dq,
                                 float* dk, float* dv, cudaStream_t s) {
  const dim3 grid(P.slots, P.Hq, P.cu ? 1 : P.B);
  const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(g);
  switch (beta_kind(P.beta)) {
    case kBetaOne:
      bwd_support_kernel<D, kBetaOne><<<grid, kBSupThreads, 0, s>>>(P, gb, delta, dq, dk, dv);
      break;
    case kBetaTwo:
      bwd_support_kernel<D, kBetaTwo><<<grid, kBSupThreads, 0, s>>>(P, gb, delta, dq, dk, dv);
      break;
    default:
      bwd_support_kernel<D, kBetaGeneral><<<grid, kBSupThreads, 0, s>>>(P, gb, delta, dq, dk,
                                                                       dv);
  }
  return cudaGetLastError();
}

template <typename T, int D, int BK>
cudaError_t launch_bwd_t(const Problem& P, const void* g, float* delta, float* dq, float* dk,
                         float* dv, cudaStream_t s) {
  const size_t smem = sizeof(BwdSmem<D>);
  auto k1 = bwd_delta_kernel<T, D, BK>;
  auto k2 = bwd_grad_kernel<T, D, BK>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(P.slots, P.Hq, P.cu ? 1 : P.B);
  k1<<<grid, kBT, smem, s>>>(P, static_cast<const T*>(g), delta);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k2<<<grid, kBT, smem, s>>>(P, static_cast<const T*>(g), delta, dq, dk, dv);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd_d(const Problem& P, const void* g, float* delta, float* dq, float* dk,
                         float* dv, cudaStream_t s) {
  switch (beta_kind(P.beta)) {
    case kBetaOne: return launch_bwd_t<T, D, kBetaOne>(P, g, delta, dq, dk, dv, s);
    case kBetaTwo: return launch_bwd_t<T, D, kBetaTwo>(P, g, delta, dq, dk, dv, s);
    default: return launch_bwd_t<T, D, kBetaGeneral>(P, g, delta, dq, dk, dv, s);
  }
}

}  // namespace

cudaError_t launch_bwd(const Problem& P, int dtype, const void* g, float* delta, float* dq,
                       float* dk, float* dv, cudaStream_t s) {
  if (P.from_support && dtype == 1) {  // the recorded tiles from their supports, then the others
    cudaError_t e = P.d == 64 ? launch_bwd_support_d<64>(P, g, delta, dq, dk, dv, s)
                              : launch_bwd_support_d<128>(P, g, delta, dq, dk, dv, s);
    if (e != cudaSuccess) return e;
  }
  if (dtype == 0)
    return P.d == 64 ? launch_bwd_d<float, 64>(P, g, delta, dq, dk, dv, s)
                     : launch_bwd_d<float, 128>(P, g, delta, dq, dk, dv, s);
  return P.d == 64 ? launch_bwd_d<__nv_bfloat16, 64>(P, g, delta, dq, dk, dv, s)
                   : launch_bwd_d<__nv_bfloat16, 128>(P, g, delta, dq, dk, dv, s);
}

}  // namespace ea
