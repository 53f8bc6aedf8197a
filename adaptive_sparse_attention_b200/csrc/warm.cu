// warm.cu -- the warm-up keys of the tensor-core tau pass: squared key norms, then per (key group,
// level) the 128 keys of largest norm among the group's first 1024 * 2^level keys, copied into a
// contiguous 128-row tile that the tau kernel loads like a key tile (see warm_level).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ea {
namespace {

constexpr int kNormThreads = 256;
constexpr int kSelectThreads = 256;

// ||k_r||^2 in fp32 for every key row r: D / 8 lanes per row, 16 bytes each.
template <int D>
__global__ void __launch_bounds__(kNormThreads) key_norms_kernel(const __nv_bfloat16* k,
                                                                 float* norms, int64_t rows) {
  constexpr int kLanes = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanes;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const int64_t row = warp * kRowsPerWarp + lane / kLanes;
  float s = 0.f;
  if (row < rows) {
    const uint4 w = reinterpret_cast<const uint4*>(k + row * D)[lane % kLanes];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(u[i] << 16), hi = __uint_as_float(u[i] & 0xffff0000u);
      s = fmaf(lo, lo, s);
      s = fmaf(hi, hi, s);
    }
  }
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (row < rows && lane % kLanes == 0) norms[row] = s;
}

// One CTA per (level, group): radix select (four 8-bit digits of the nonnegative fp32 norm) of
// the 128th largest norm in the level's range, then the 128 rows -- every key above it and as
// many keys equal to it as needed -- copied to the level's warm tile.  Levels whose range is
// wider than any query tile of the group may use are skipped.
template <int D>
__global__ void __launch_bounds__(kSelectThreads) warm_select_kernel(Problem P) {
  const int level = blockIdx.x, grp = blockIdx.y;
  const int s = grp / P.Hkv, kvh = grp - s * P.Hkv;
  int64_t base;
  int seq_len;
  if (P.cu == nullptr) {
    base = static_cast<int64_t>(grp) * P.T;
    seq_len = P.T;
  } else {
    base = static_cast<int64_t>(kvh) * P.T + P.cu[s];
    seq_len = P.cu[s + 1] - P.cu[s];
  }
  const int usable = P.causal ? kTile * ((seq_len + kTile - 1) / kTile - 1) : seq_len;
  const int n = kWarmBase << level;
  if (n > usable) return;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(P.norms + base);

  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need, s_gt, s_eq;
  __shared__ int idx[kTile];
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0;
  int need = kTile;  // keys still to take at or below the current prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kSelectThreads) {
      const uint32_t u = bits[i];
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      int acc = 0, dsel = 0;
      for (int b = 255; b >= 0; --b) {
        const int h = static_cast<int>(hist[b]);
        if (acc + h >= need) {
          dsel = b;
          break;
        }
        acc += h;
      }
      s_prefix = prefix | (static_cast<uint32_t>(dsel) << shift);
      s_need = need - acc;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 255u << shift;
  }
  // prefix: the bits of the 128th largest norm; kTile - need keys lie strictly above it
  if (tid == 0) {
    s_gt = 0;
    s_eq = 0;
  }
  __syncthreads();
  for (int i = tid; i < n; i += kSelectThreads) {
    const uint32_t u = bits[i];
    if (u > prefix) {
      idx[atomicAdd(&s_gt, 1)] = i;
    } else if (u == prefix) {
      const int e = atomicAdd(&s_eq, 1);
      if (e < need) idx[kTile - need + e] = i;
    }
  }
  __syncthreads();
  // copy: D / 8 lanes of 16 bytes per row
  constexpr int kLanes = D / 8;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(P.k) +
                                                    base * D);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.warm) +
                                        (static_cast<int64_t>(grp) * P.warm_levels + level) *
                                            kTile * D);
  for (int e = tid; e < kTile * kLanes; e += kSelectThreads) {
    const int r = e / kLanes, c = e - r * kLanes;
    dst[static_cast<int64_t>(r) * kLanes + c] = src[static_cast<int64_t>(idx[r]) * kLanes + c];
  }
}

template <int D>
cudaError_t launch_warm_t(const Problem& P, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hkv * P.T;
  constexpr int kRowsPerBlock = (kNormThreads / 32) * (32 / (D / 8));
  const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  key_norms_kernel<D><<<static_cast<unsigned>(blocks), kNormThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(P.k), P.norms, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int groups = P.B * P.Hkv;  // batches or sequences x kv heads
  warm_select_kernel<D><<<dim3(P.warm_levels, groups), kSelectThreads, 0, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_warm(const Problem& P, cudaStream_t s) {
  if (P.warm_levels <= 0) return cudaSuccess;
  return P.d == 64 ? launch_warm_t<64>(P, s) : launch_warm_t<128>(P, s);
}

}  // namespace ea
