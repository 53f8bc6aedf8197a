// simt.cu -- CUDA-core kernels of the entmax attention forward pass.
//
//   tau_simt_kernel      single sweep over the key tiles of a query tile: scores in true fp32,
//                        candidate buffers, Halley + bisection per row, block mask + compact
//                        list.  The path for fp32 inputs.
//   tau_fallback_kernel  the multi-sweep search for query tiles whose candidate buffers
//                        overflowed: one sweep for the row max, one per search step over all
//                        valid keys (from the main pass's tau, until every row has settled),
//                        one for the mask bits.  Any dtype.
//   out_simt_kernel      output pass on the CUDA cores over the listed key tiles.
//
// One CTA of 128 threads per query tile, thread r owning row r of the tile.  The query tile
// sits in shared memory as fp32 (padded rows); keys and values stream through shared memory in
// chunks of 32, widened to fp32.  Each chunk's 32 x 128 scores go to shared memory, column r
// belonging to thread r.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace ea {
namespace {

constexpr int kChunk = 32;
constexpr int kThreads = 128;

template <int D>
struct SimtSmem {
  static constexpr int QS = D + 4;  // padded query row: conflict-free float4 reads
  float qs[kTile * QS];
  float ks[kChunk * D];
  float vs[kChunk * D];
  float xs[kChunk * kTile];  // scores of the current chunk, [key][row]
};

template <typename T>
__device__ __forceinline__ const T* as(const void* p) { return static_cast<const T*>(p); }

// Loads rows [j0, j0 + 32) of a key or value head (rows past len as zero) into dst[32][D].
template <typename T, int D>
__device__ __forceinline__ void load_chunk(const T* base, int64_t row0, int j0, int len,
                                           float* dst, int tid) {
  for (int i = tid; i < kChunk * D; i += kThreads) {
    const int jj = i / D, c = i % D;
    dst[i] = (j0 + jj < len) ? load_elem(base, (row0 + j0 + jj) * D + c) : 0.f;
  }
}

template <typename T, int D>
__device__ __forceinline__ void load_q_tile(const Problem& P, const TileInfo& t, float* qs,
                                            int tid) {
  const T* qp = as<T>(P.q);
  for (int i = tid; i < kTile * D; i += kThreads) {
    const int r = i / D, c = i % D;
    qs[r * SimtSmem<D>::QS + c] =
        (r < t.nrows) ? load_elem(qp, (t.qhead + t.seq_start + t.row0 + r) * D + c) : 0.f;
  }
}

// Scores of thread tid's row against the 32 keys of the chunk, masked to -inf outside the row's
// valid key range (past the sequence end; past the row's own position when causal; all keys for
// rows past the tile end).  Written to xs[jj * 128 + tid].
template <int D>
__device__ __noinline__ void chunk_scores(const float* qs, const float* ks, float* xs, int tid,
                                          int j0, int jmax) {
  const float4* q4 = reinterpret_cast<const float4*>(qs + tid * SimtSmem<D>::QS);
  const float4* k4 = reinterpret_cast<const float4*>(ks);
#pragma unroll 2
  for (int jj = 0; jj < kChunk; ++jj) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int c4 = 0; c4 < D / 4; c4 += 2) {
      const float4 qa = q4[c4], qb = q4[c4 + 1];
      const float4 u = k4[jj * (D / 4) + c4], w = k4[jj * (D / 4) + c4 + 1];
      a0 = fmaf(qa.x, u.x, a0);
      a0 = fmaf(qa.y, u.y, a0);
      a0 = fmaf(qa.z, u.z, a0);
      a0 = fmaf(qa.w, u.w, a0);
      a1 = fmaf(qb.x, w.x, a1);
      a1 = fmaf(qb.y, w.y, a1);
      a1 = fmaf(qb.z, w.z, a1);
      a1 = fmaf(qb.w, w.w, a1);
    }
    xs[jj * kTile + tid] = (j0 + jj < jmax) ? a0 + a1 : -INFINITY;
  }
}

// Valid keys of thread tid's row: [0, jmax); 0 for rows past the end of the tile.
__device__ __forceinline__ int row_jmax(const Problem& P, const TileInfo& t, int tid) {
  if (tid >= t.nrows) return 0;
  return P.causal ? t.row0 + tid + 1 : t.seq_len;
}

// Runs fn(kt) after the scores of each 32-key chunk of the tile's key range are in sm.xs.
template <typename T, int D, typename Fn>
__device__ __forceinline__ void sweep_keys(const Problem& P, const TileInfo& t, SimtSmem<D>& sm,
                                           int tid, Fn&& fn) {
  const T* kp = as<T>(P.k);
  const int jmax = row_jmax(P, t, tid);
  for (int kt = 0; kt < t.nkt; ++kt) {
    for (int ch = 0; ch < kTile / kChunk; ++ch) {
      const int j0 = kt * kTile + ch * kChunk;
      if (j0 >= t.seq_len) break;
      __syncthreads();
      load_chunk<T, D>(kp, t.khead + t.seq_start, j0, t.seq_len, sm.ks, tid);
      __syncthreads();
      chunk_scores<D>(sm.qs, sm.ks, sm.xs, tid, j0, jmax);
      fn(kt);
    }
  }
}

template <typename T, int D, int BK>
__global__ void __launch_bounds__(kThreads) tau_simt_kernel(Problem P) {
  extern __shared__ __align__(16) unsigned char smem[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem);
  CandSmem& cs = *reinterpret_cast<CandSmem*>(smem + sizeof(SimtSmem<D>));
  const int tid = threadIdx.x;
  const int slot = gridDim.x - 1 - blockIdx.x;  // longest query tiles first
  const TileInfo t = map_tile(P, slot, blockIdx.y, blockIdx.z);
  if (!t.valid) {
    emit_empty(P, t, tid, kThreads);
    return;
  }
  for (int w = tid; w < kMaxWords; w += kThreads) cs.words[w] = 0u;
  cs.rowmax[tid] = -INFINITY;  // kThreads == kTile: thread tid owns row tid
  if (tid == 0) cs.fallback = P.force_fallback;
  load_q_tile<T, D>(P, t, sm.qs, tid);

  // chunk g (keys 32 g .. 32 g + 31) of every key tile is segment g
  static_assert(kSeg * kChunk == kTile, "one 32-key chunk per segment");
  RowCand rc0, rc1, rc2, rc3;
  rc0.init(1.f / P.c);
  rc1.init(1.f / P.c);
  rc2.init(1.f / P.c);
  rc3.init(1.f / P.c);
  int chunk = 0;
  sweep_keys<T, D>(P, t, sm, tid, [&](int kt) {
    float x[kChunk];
#pragma unroll
    for (int jj = 0; jj < kChunk; ++jj) x[jj] = sm.xs[jj * kTile + tid];
    switch (chunk++ & 3) {  // uniform across the block
      case 0:
        feed_warp<kChunk>(rc0, cs, cs.xrow[tid >> 5], tid, tid, tid & 31, x, kt);
        break;
      case 1:
        feed_warp<kChunk>(rc1, cs, cs.xrow[tid >> 5], kTile + tid, tid, tid & 31, x, kt);
        break;
      case 2:
        feed_warp<kChunk>(rc2, cs, cs.xrow[tid >> 5], 2 * kTile + tid, tid, tid & 31, x, kt);
        break;
      default:
        feed_warp<kChunk>(rc3, cs, cs.xrow[tid >> 5], 3 * kTile + tid, tid, tid & 31, x, kt);
        break;
    }
  });
  rc0.publish(cs, tid);
  rc1.publish(cs, kTile + tid);
  rc2.publish(cs, 2 * kTile + tid);
  rc3.publish(cs, 3 * kTile + tid);
  __syncthreads();
  solve_rows<BK>(P, t, cs, tid, kThreads);
  __syncthreads();
  if (tid < 32) emit_tile(P, t, cs.words, cs.fallback, tid);
}

template <typename T, int D, int BK>
__global__ void __launch_bounds__(kThreads) tau_fallback_kernel(Problem P) {
  extern __shared__ __align__(16) unsigned char smem[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem);
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + sizeof(SimtSmem<D>));
  const int tid = threadIdx.x;
  const int ntiles = (P.cu ? 1 : P.B) * P.Hq * P.slots;
  const int nq = min(*P.queue_count, ntiles);
  for (int i = blockIdx.x; i < nq; i += gridDim.x) {
    const int id = P.queue[i];
    if (id < 0 || id >= ntiles) continue;  // uniform across the block
    const int slot = id % P.slots;
    const int h = (id / P.slots) % P.Hq;
    const int b = id / (P.slots * P.Hq);
    const TileInfo t = map_tile(P, slot, h, b);
    __syncthreads();
    for (int w = tid; w < kMaxWords; w += kThreads) words[w] = 0u;
    load_q_tile<T, D>(P, t, sm.qs, tid);
    const bool row_ok = tid < t.nrows;
    const int pos = t.row0 + tid;

    float m = -INFINITY;  // raw
    sweep_keys<T, D>(P, t, sm, tid, [&](int) {
      for (int jj = 0; jj < kChunk; ++jj) m = fmaxf(m, sm.xs[jj * kTile + tid]);
    });
    const float mz = row_ok ? P.c * m : 0.f;
    const int n = row_ok ? (P.causal ? pos + 1 : t.seq_len) : 1;
    Search sr;
    sr.init(mz, n, P.alpha);
    {  // start from the tau the main pass found on the candidates it kept (inside the bracket)
      const float t_kept = row_ok ? P.tau[t.qhead + t.seq_start + pos] : sr.lo;
      if (t_kept > sr.lo && t_kept < sr.hi) sr.tau = t_kept;
    }
    for (int it = 0; it < P.n_iter; ++it) {
      // stop once every row of the tile has settled (uniform across the block)
      if (it > 0 && !__syncthreads_or(row_ok && !sr.settled())) break;
      const float tau = sr.tau;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f;
      sweep_keys<T, D>(P, t, sm, tid, [&](int) {
        for (int jj = 0; jj < kChunk; ++jj) {
          const float y = P.c * sm.xs[jj * kTile + tid] - tau;
          if (y > 0.f) {
            float a, bb, cc;
            entmax_powers<BK>(y, P.beta, a, bb, cc);
            s0 += a;
            s1 += bb;
            s2 += cc;
          }
        }
      });
      sr.step<BK>(s0, s1, s2, P.beta);
    }
    const float tau = sr.tau;
    if (row_ok) P.tau[t.qhead + t.seq_start + pos] = tau;
    sweep_keys<T, D>(P, t, sm, tid, [&](int kt) {
      bool any = false;
      for (int jj = 0; jj < kChunk; ++jj) any |= (P.c * sm.xs[jj * kTile + tid] > tau);
      if (any) atomicOr(&words[kt >> 5], 1u << (kt & 31));
    });
    __syncthreads();
    if (tid < 32) emit_tile(P, t, words, 0, tid);
  }
}

template <typename T, int D, int BK>
__global__ void __launch_bounds__(kThreads) out_simt_kernel(Problem P) {
  extern __shared__ __align__(16) unsigned char smem[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem);
  const int tid = threadIdx.x;
  const int slot = gridDim.x - 1 - blockIdx.x;
  const TileInfo t = map_tile(P, slot, blockIdx.y, blockIdx.z);
  if (!t.valid) return;
  if (P.from_support && P.pending[t.tile_id] == 0) return;  // o from the tile's support list
  const T* kp = as<T>(P.k);
  const T* vp = as<T>(P.v);
  load_q_tile<T, D>(P, t, sm.qs, tid);
  const bool row_ok = tid < t.nrows;
  const int pos = t.row0 + tid;
  const int jmax = row_jmax(P, t, tid);
  const float tau = row_ok ? P.tau[t.qhead + t.seq_start + pos] : INFINITY;
  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.f;

  const int cnt = list_count(P, t);  // see clamp_kt
  const int* list = P.list + t.tile_id * P.nkt_max;
  for (int i = 0; i < cnt; ++i) {
    const int kt = list_tile(P, list, i, t.nkt);
    for (int ch = 0; ch < kTile / kChunk; ++ch) {
      const int j0 = kt * kTile + ch * kChunk;
      if (j0 >= t.seq_len) break;
      __syncthreads();
      load_chunk<T, D>(kp, t.khead + t.seq_start, j0, t.seq_len, sm.ks, tid);
      load_chunk<T, D>(vp, t.khead + t.seq_start, j0, t.seq_len, sm.vs, tid);
      __syncthreads();
      chunk_scores<D>(sm.qs, sm.ks, sm.xs, tid, j0, jmax);
      for (int jj = 0; jj < kChunk; ++jj) {
        const float p = entmax_p<BK>(P.c * sm.xs[jj * kTile + tid] - tau, P.beta);
        if (p > 0.f) {
          const float4* v4 = reinterpret_cast<const float4*>(sm.vs + jj * D);
#pragma unroll
          for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 vv = v4[c4];
            o[4 * c4 + 0] = fmaf(p, vv.x, o[4 * c4 + 0]);
            o[4 * c4 + 1] = fmaf(p, vv.y, o[4 * c4 + 1]);
            o[4 * c4 + 2] = fmaf(p, vv.z, o[4 * c4 + 2]);
            o[4 * c4 + 3] = fmaf(p, vv.w, o[4 * c4 + 3]);
          }
        }
      }
    }
  }
  if (row_ok) {
    T* op = static_cast<T*>(P.out);
    const int64_t row = t.qhead + t.seq_start + pos;
#pragma unroll
    for (int c = 0; c < D; ++c) store_elem(op, row * D + c, o[c]);
  }
}

dim3 tile_grid(const Problem& P) { return dim3(P.slots, P.Hq, P.cu ? 1 : P.B); }

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D, int BK>
cudaError_t launch_tau_simt_t(const Problem& P, cudaStream_t s) {
  const size_t smem = sizeof(SimtSmem<D>) + sizeof(CandSmem);
  auto kern = tau_simt_kernel<T, D, BK>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<tile_grid(P), kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

template <typename T, int D, int BK>
cudaError_t launch_out_simt_t(const Problem& P, cudaStream_t s) {
  const size_t smem = sizeof(SimtSmem<D>);
  auto kern = out_simt_kernel<T, D, BK>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<tile_grid(P), kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

template <typename T, int D, int BK>
cudaError_t launch_fallback_t(const Problem& P, int num_ctas, cudaStream_t s) {
  const size_t smem = sizeof(SimtSmem<D>) + kMaxWords * sizeof(uint32_t);
  auto kern = tau_fallback_kernel<T, D, BK>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<num_ctas, kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

// dtype x d x beta-kind dispatch
#define EA_DISPATCH(FN, ...)                                                           \
  do {                                                                                 \
    const int bk = beta_kind(P.beta);                                                  \
    if (dtype == 0) {                                                                  \
      if (P.d == 64) {                                                                 \
        if (bk == kBetaOne) return FN<float, 64, kBetaOne>(__VA_ARGS__);               \
        if (bk == kBetaTwo) return FN<float, 64, kBetaTwo>(__VA_ARGS__);               \
        return FN<float, 64, kBetaGeneral>(__VA_ARGS__);                               \
      }                                                                                \
      if (bk == kBetaOne) return FN<float, 128, kBetaOne>(__VA_ARGS__);                \
      if (bk == kBetaTwo) return FN<float, 128, kBetaTwo>(__VA_ARGS__);                \
      return FN<float, 128, kBetaGeneral>(__VA_ARGS__);                                \
    }                                                                                  \
    if (P.d == 64) {                                                                   \
      if (bk == kBetaOne) return FN<__nv_bfloat16, 64, kBetaOne>(__VA_ARGS__);         \
      if (bk == kBetaTwo) return FN<__nv_bfloat16, 64, kBetaTwo>(__VA_ARGS__);         \
      return FN<__nv_bfloat16, 64, kBetaGeneral>(__VA_ARGS__);                         \
    }                                                                                  \
    if (bk == kBetaOne) return FN<__nv_bfloat16, 128, kBetaOne>(__VA_ARGS__);          \
    if (bk == kBetaTwo) return FN<__nv_bfloat16, 128, kBetaTwo>(__VA_ARGS__);          \
    return FN<__nv_bfloat16, 128, kBetaGeneral>(__VA_ARGS__);                          \
  } while (0)

}  // namespace

cudaError_t launch_tau_simt(const Problem& P, int dtype, cudaStream_t s) {
  EA_DISPATCH(launch_tau_simt_t, P, s);
}

cudaError_t launch_tau_fallback(const Problem& P, int dtype, int num_ctas, cudaStream_t s) {
  EA_DISPATCH(launch_fallback_t, P, num_ctas, s);
}

cudaError_t launch_out_simt(const Problem& P, int dtype, cudaStream_t s) {
  EA_DISPATCH(launch_out_simt_t, P, s);
}

}  // namespace ea
