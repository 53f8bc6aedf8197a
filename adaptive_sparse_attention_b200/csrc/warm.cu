// warm.cu -- the warm-up keys of the tensor-core tau pass: squared key norms, then per (key group,
// level) the 128 keys of largest norm among the group's first 1024 * 2^level keys, copied into a
// contiguous 128-row tile that the tau kernel loads like a key tile (see warm_level).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ea {
namespace {

constexpr int kNormThreads = 256;
constexpr int kSelectThreads = 1024;
static_assert(kWarmBase % kSelectThreads == 0, "every level's range is a whole number of CTA rows");

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

// Adds 1 to hist[bin] for every lane with bin < 256, one shared-memory atomic per distinct bin
// of the warp: the norms of a key range share their leading bits, so most lanes of a warp hit
// the same bin in the first digits.  Call with the whole warp.
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t bin, int lane) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// One CTA per (level, group): radix select (four 8-bit digits of the nonnegative fp32 norm) of
// the 128th largest norm in the level's range, then the 128 rows -- every key above it and as
// many keys equal to it as needed -- copied to the level's warm tile.  Levels whose range is
// wider than any query tile of the group may use are skipped.  The range holds 1024 * 2^level
// keys, a multiple of the CTA size, so every warp runs the same number of loop trips.
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
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t prefix = 0, mask = 0;
  int need = kTile;  // keys still to take at or below the current prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += 4 * kSelectThreads) {  // four loads in flight per thread
      uint32_t u[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        u[e] = i + e * kSelectThreads < n ? bits[i + e * kSelectThreads] : 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i + e * kSelectThreads < n)  // the same for the whole warp
          warp_hist_add(hist, (u[e] & mask) == prefix ? (u[e] >> shift) & 255u : 256u, lane);
    }
    __syncthreads();
    if (tid < 32) {  // the digit that holds the need-th largest key, by warp 0
      // lane l owns bins 8 l .. 8 l + 7; above = keys in the bins of lanes above l
      int h[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = static_cast<int>(hist[8 * lane + j]);
        sum += h[j];
      }
      int incl = sum;  // keys in bins >= 8 l
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += t;
      }
      int acc = incl - sum;
      if (acc < need && incl >= need) {  // exactly one lane
        int dsel = 8 * lane;
        for (int j = 7; j >= 0; --j) {
          if (acc + h[j] >= need) {
            dsel = 8 * lane + j;
            break;
          }
          acc += h[j];
        }
        s_prefix = prefix | (static_cast<uint32_t>(dsel) << shift);
        s_need = need - acc;
      }
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
      const int k = atomicAdd(&s_eq, 1);
      if (k < need) idx[kTile - need + k] = i;
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
