// screen.cu -- FP8 screening of the key tiles the tau pass must score in bf16.
//
// The tau pass needs, per row i, every key with z_ij > m_i - 1 (m_i = max_j z_ij, z = c q.k,
// c = (alpha - 1) / sqrt(d)).  A key tile none of whose pairs can reach that window contributes
// no candidate and does not hold the row max, so the bf16 pass may skip it and still find the
// same tau, mask and supports.  The screen decides this from fp8 (e4m3) products with a rigorous
// error bound:
//   q_i = s_i q8_i + eq_i       (s_i = max|q_i| / 448 per row, q8 = e4m3(q / s))
//   k_j = S_t k8_j + ek_j       (S_t = max|k| / 448 per 128-key tile t, k8 = e4m3(k / S_t))
//   |q_i . k_j - s_i S_t q8_i . k8_j| <= |eq_i| |k_j| + |s_i q8_i| |ek_j|         (Cauchy-Schwarz)
//                                     <= |eq_i| Kmax_t + nq_i Emax_t             (tile maxima)
// plus the fp32 accumulation of the product (below).  With r8_ij = s_i S_t q8_i . k8_j and
// b_it the bound, every raw score of row i in tile t lies in [r8_ij - b_it, r8_ij + b_it].  While
// it sweeps the key tiles of a query tile in order, the screen keeps per row a lower bound
// L_i <= m_i (the largest c (r8_ij - b_it) so far, over the row's valid keys) and marks tile t
// needed if some row has c (max_j r8_ij + b_it) > L_i - 1.  An unmarked tile has z_ij <= m_i - 1
// for every pair: no candidate, and not the row max (which would make the tile marked).
//
//   screen_prep_q_kernel  one warp per query row: q8 row, (s_i, |eq_i|, nq_i = |s_i q8_i|).
//   screen_prep_k_kernel  one CTA per key tile: k8 rows, (S_t, Kmax_t, Emax_t).
//   screen_kernel         persistent like the tau kernel (16 score warps, 1 TMA warp, 1 MMA warp,
//                         four TMEM score buffers): kind::f8f6f4 products S8 = q8 k8^T, the test
//                         above per row and key tile, and per query tile the ascending list of
//                         needed key tiles and its count, which the tau kernel then visits.
// d = 128 only (a 128-byte e4m3 row is one 128-byte swizzle row).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace ea {
namespace {

constexpr float kE4m3Max = 448.f;
// fp32 accumulation of the fp8 product, relative to nq_i Kmax_t: the tensor core sums 128
// exact fp8 products; 2^-9 covers a reduced-precision internal accumulation with a wide margin.
constexpr float kAccRel = 1.f / 512.f;
constexpr int kScrScoreWarps = 16;
constexpr int kScrThreads = 32 * (kScrScoreWarps + 2);
constexpr int kScrStages = 4;
constexpr int kScrSBufs = 4;
constexpr int kScrTmaWarp = kScrScoreWarps;
constexpr int kScrMmaWarp = kScrScoreWarps + 1;

__device__ __forceinline__ float e4m3_round(float x, uint8_t* byte) {
  const __nv_fp8_e4m3 v(x);  // round to nearest, saturating to the finite range
  *byte = v.__x;
  return static_cast<float>(v);
}

// ---------------------------------------------------------------------------------- prep ----
template <int D>
__global__ void __launch_bounds__(256) screen_prep_q_kernel(const __nv_bfloat16* __restrict__ q,
                                                            int64_t rows, uint8_t* __restrict__ q8,
                                                            float4* __restrict__ qst) {
  constexpr int kPer = D / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < rows; row += warps) {
    float x[kPer];
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      x[e] = __bfloat162float(q[row * D + lane * kPer + e]);
      mx = fmaxf(mx, fabsf(x[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float s = mx > 0.f ? mx / kE4m3Max : 1.f;
    const float inv = 1.f / s;
    float e2 = 0.f, n2 = 0.f;
    uint32_t packed = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      uint8_t b;
      const float d = s * e4m3_round(x[e] * inv, &b);
      packed |= static_cast<uint32_t>(b) << (8 * e);
      e2 = fmaf(x[e] - d, x[e] - d, e2);
      n2 = fmaf(d, d, n2);
    }
    if (kPer == 4) {
      reinterpret_cast<uint32_t*>(q8 + row * D)[lane] = packed;
    } else {
#pragma unroll
      for (int e = 0; e < kPer; ++e) q8[row * D + lane * kPer + e] = (packed >> (8 * e)) & 0xffu;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      e2 += __shfl_xor_sync(0xffffffffu, e2, o);
      n2 += __shfl_xor_sync(0xffffffffu, n2, o);
    }
    // the error norm rounded up a little: the sums themselves carry fp32 rounding
    if (lane == 0) qst[row] = make_float4(s, sqrtf(e2) * 1.0001f + 1e-30f, sqrtf(n2) * 1.0001f, 0.f);
  }
}

// Key-tile id of key tile kt of tile t's key group (the layout of the key-tile statistics):
// fixed length ((b Hkv + hk) nkt_max + kt), packed (hk S + slot of the sequence's first tile + kt).
__device__ __forceinline__ int64_t key_tile_id(const Problem& P, const TileInfo& t, int kt) {
  if (P.cu == nullptr) return static_cast<int64_t>(t.grp) * P.nkt_max + kt;
  const int seq = t.grp / P.Hkv, hk = t.grp % P.Hkv;
  return static_cast<int64_t>(hk) * P.slots + t.seq_start / kTile + seq + kt;
}

// One CTA of 128 threads per (key group, key tile): thread j owns key row j of the tile.
template <int D>
__global__ void __launch_bounds__(128) screen_prep_k_kernel(Problem P, uint8_t* __restrict__ k8,
                                                            float4* __restrict__ kst) {
  __shared__ float red[2][4];
  // the key tile as query-tile slot `slot` of the first query head of kv head blockIdx.y
  const TileInfo t = map_tile(P, blockIdx.x, blockIdx.y * P.G, blockIdx.z);
  if (!t.valid) return;
  const int kt = t.qt, j = threadIdx.x;
  const bool ok = kt * kTile + j < t.seq_len;
  const int64_t row = t.khead + t.seq_start + static_cast<int64_t>(kt) * kTile + j;
  const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(P.k) + row * D;
  float mx = 0.f;
  if (ok)
    for (int e = 0; e < D; ++e) mx = fmaxf(mx, fabsf(__bfloat162float(kr[e])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((j & 31) == 0) red[0][j >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  const float s = mx > 0.f ? mx / kE4m3Max : 1.f;
  const float inv = 1.f / s;
  float e2 = 0.f, k2 = 0.f;
  if (ok) {
    for (int e = 0; e < D; e += 4) {
      uint32_t packed = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x = __bfloat162float(kr[e + u]);
        uint8_t b;
        const float d = s * e4m3_round(x * inv, &b);
        packed |= static_cast<uint32_t>(b) << (8 * u);
        e2 = fmaf(x - d, x - d, e2);
        k2 = fmaf(x, x, k2);
      }
      reinterpret_cast<uint32_t*>(k8 + row * D)[e / 4] = packed;
    }
  }
  float en = sqrtf(e2), kn = sqrtf(k2);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    en = fmaxf(en, __shfl_xor_sync(0xffffffffu, en, o));
    kn = fmaxf(kn, __shfl_xor_sync(0xffffffffu, kn, o));
  }
  __syncthreads();
  if ((j & 31) == 0) {
    red[0][j >> 5] = kn;
    red[1][j >> 5] = en;
  }
  __syncthreads();
  if (j == 0) {
    kn = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
    en = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
    kst[key_tile_id(P, t, kt)] = make_float4(s, kn * 1.0001f, en * 1.0001f + 1e-30f, 0.f);
  }
}

// --------------------------------------------------------------------------- screen kernel ----
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (format code 0), fp32 accumulate,
// both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

struct ScreenSmem {
  alignas(1024) uint8_t q[kTile * 128];
  alignas(1024) uint8_t k[kScrStages][kTile * 128];
  float lb[kTile];  // per row: largest lower bound of the row's z found so far
  uint32_t words[kMaxWords];
  int wbase[kMaxWords];
  uint64_t q_full, q_empty;
  uint64_t k_full[kScrStages], k_empty[kScrStages];
  uint64_t s_full[kScrSBufs], s_empty[kScrSBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void scr_score_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kScrScoreWarps) : "memory");
}

__global__ void __launch_bounds__(kScrThreads, 1)
    screen_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  Problem P, const float4* __restrict__ qst, const float4* __restrict__ kst,
                  int* __restrict__ list, int* __restrict__ count) {
  extern __shared__ unsigned char smem_raw[];
  ScreenSmem& sm = *reinterpret_cast<ScreenSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per_slot = P.Hq * (P.cu ? 1 : P.B);
  const int ntiles = P.slots * per_slot;
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * 128;
  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kScrStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int b = 0; b < kScrSBufs; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_empty[b], kScrScoreWarps);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int w = tid; w < kMaxWords; w += kScrThreads) sm.words[w] = 0u;
  if (warp == kScrMmaWarp) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kScrTmaWarp) {
    if (lane == 0) {
      int it = 0, gk = 0;
      bool ok = true;
      for (int L = blockIdx.x; ok && L < ntiles; L += gridDim.x) {
        const TileInfo t = tau_tile(P, L, per_slot);
        if (!t.valid) continue;
        if (it > 0 && !mbar_wait(&sm.q_empty, (it - 1) & 1, abort, P.status)) break;
        mbar_expect_tx(&sm.q_full, kTileBytes);
        tma_load_2d(sm.q, &tmq, &sm.q_full, 0, static_cast<int>(t.qhead + t.seq_start + t.row0));
        ++it;
        const int krow0 = static_cast<int>(t.khead + t.seq_start);
        for (int kt = 0; kt < t.nkt; ++kt, ++gk) {
          const int s = gk % kScrStages;
          if (gk >= kScrStages &&
              !mbar_wait(&sm.k_empty[s], ((gk / kScrStages) - 1) & 1, abort, P.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&sm.k_full[s], kTileBytes);
          tma_load_2d(sm.k[s], &tmk, &sm.k_full[s], 0, krow0 + kt * kTile);
        }
      }
      for (int g = (gk > kScrStages ? gk - kScrStages : 0); g < gk; ++g)
        mbar_wait(&sm.k_full[g % kScrStages], (g / kScrStages) & 1, abort, P.status);
      if (it > 0) mbar_wait(&sm.q_full, (it - 1) & 1, abort, P.status);
    }
  } else if (warp == kScrMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3(128, 128);
      int it = 0, gk = 0;
      bool ok = true;
      for (int L = blockIdx.x; ok && L < ntiles; L += gridDim.x) {
        const TileInfo t = tau_tile(P, L, per_slot);
        if (!t.valid) continue;
        if (!mbar_wait(&sm.q_full, it & 1, abort, P.status)) break;
        ++it;
        for (int kt = 0; kt < t.nkt; ++kt, ++gk) {
          const int s = gk % kScrStages, b = gk % kScrSBufs;
          if (!mbar_wait(&sm.k_full[s], (gk / kScrStages) & 1, abort, P.status) ||
              (gk >= kScrSBufs &&
               !mbar_wait(&sm.s_empty[b], ((gk / kScrSBufs) - 1) & 1, abort, P.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k32 = 0; k32 < 4; ++k32)  // 32 e4m3 values = 32 bytes of K per product
            mma_ss_f8(tmem + static_cast<uint32_t>(b * 128),
                      kmajor_desc(smem_u32(sm.q), kTile, k32),
                      kmajor_desc(smem_u32(sm.k[s]), kTile, k32), idesc, k32 > 0 ? 1u : 0u);
          mma_commit(&sm.k_empty[s]);
          mma_commit(&sm.s_full[b]);
        }
        if (ok) mma_commit(&sm.q_empty);
      }
      if (gk > 0) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, abort, P.status);
      }
    }
  } else {  // score warps 0..15: warp w reads TMEM lanes 32 (w % 4) .., segment w / 4
    const int quarter = warp & 3, seg = warp >> 2;
    const int r = quarter * 32 + lane;
    int gs = 0;
    for (int L = blockIdx.x; L < ntiles; L += gridDim.x) {
      const TileInfo t = tau_tile(P, L, per_slot);
      if (!t.valid) {
        if (tid == 0) count[t.tile_id] = 0;
        continue;
      }
      if (tid < kTile) sm.lb[tid] = -INFINITY;
      scr_score_sync();
      if (tid < kMaxWords) sm.words[tid] = 0u;
      const bool row_ok = r < t.nrows;
      const int jmax = row_ok ? (P.causal ? t.row0 + r + 1 : t.seq_len) : 0;
      const float4 qs = row_ok ? qst[t.qhead + t.seq_start + t.row0 + r] : make_float4(0, 0, 0, 0);
      scr_score_sync();  // the words are clear before any warp marks a tile
      float lbr = -INFINITY;  // this thread's copy of its row's lower bound
      bool aborted = false;
      for (int kt = 0; kt < t.nkt; ++kt, ++gs) {
        const int b = gs % kScrSBufs;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&sm.s_full[b], (gs / kScrSBufs) & 1, abort, P.status))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        float x[32];
        tmem_row32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                       static_cast<uint32_t>(b * 128 + seg * 32),
                   kt * kTile + seg * 32, jmax, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_empty[b]);
        const float cmax = fmaxf(max16(x, 0), max16(x, 16));
        bool need = false;
        if (cmax > -INFINITY) {
          const float4 ks = kst[key_tile_id(P, t, kt)];
          const float r8 = qs.x * ks.x * cmax;                        // max_j of s_i S_t q8 . k8
          const float bnd = fmaf(qs.y, ks.y, qs.z * ks.z) + kAccRel * qs.z * ks.y;
          const float lo = P.c * (r8 - bnd), hi = P.c * (r8 + bnd);
          const float shared_lb = *reinterpret_cast<volatile float*>(&sm.lb[r]);
          lbr = fmaxf(lbr, fmaxf(shared_lb, lo));
          if (lo > shared_lb) sm.lb[r] = lo;  // publish to the row's other segments
          need = hi > lbr - 1.f;
        }
        if (__any_sync(0xffffffffu, need) && lane == 0)
          atomicOr(&sm.words[kt >> 5], 1u << (kt & 31));
      }
      scr_score_sync();
      // the tile's list: ascending needed key tiles and their count
      if (warp == 0) {
        int base = 0;
        for (int w0 = 0; w0 < P.W; w0 += 32) {
          const int w = w0 + lane;
          const int c = (w < P.W) ? __popc(sm.words[w]) : 0;
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (w < P.W) sm.wbase[w] = base + incl - c;
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) count[t.tile_id] = base;
      }
      scr_score_sync();
      int* out = list + t.tile_id * P.nkt_max;
      for (int i = tid; i < P.W * 32; i += 32 * kScrScoreWarps) {
        const uint32_t bits = sm.words[i >> 5];
        const uint32_t bit = 1u << (i & 31);
        if (bits & bit) out[sm.wbase[i >> 5] + __popc(bits & (bit - 1u))] = i;
      }
      if (aborted) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kScrMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_screen(const Problem& P0, void* q8, void* qst, void* k8, void* kst, int* list,
                          int* count, cudaStream_t s) {
  Problem P = P0;
  // the tau kernel's query-tile order (key-group-major when the keys exceed L2)
  P.kv_major = static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hkv * P.T * P.d * 2 > (96ll << 20) ? 1 : 0;
  const int64_t qrows = static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hq * P.T;
  const int64_t krows = static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hkv * P.T;
  screen_prep_q_kernel<128><<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(P.q), qrows,
                                                static_cast<uint8_t*>(q8),
                                                static_cast<float4*>(qst));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  screen_prep_k_kernel<128><<<dim3(P.slots, P.Hkv, P.cu ? 1 : P.B), 128, 0, s>>>(
      P, static_cast<uint8_t*>(k8), static_cast<float4*>(kst));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk;
  e = make_map_u8(&mq, q8, qrows, 128);
  if (e == cudaSuccess) e = make_map_u8(&mk, k8, krows, 128);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(ScreenSmem) + 1024;
  e = cudaFuncSetAttribute(screen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = device_sms(&sms);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = static_cast<int64_t>(P.slots) * P.Hq * (P.cu ? 1 : P.B);
  screen_kernel<<<static_cast<unsigned>(std::min<int64_t>(ntiles, sms)), kScrThreads, smem, s>>>(
      mq, mk, P, static_cast<const float4*>(qst), static_cast<const float4*>(kst), list, count);
  return cudaGetLastError();
}

}  // namespace ea
