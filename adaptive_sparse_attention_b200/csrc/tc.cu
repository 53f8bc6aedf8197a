// tc.cu -- tensor-core (tcgen05) kernels of the entmax attention forward pass, bf16, sm_100a.
//
// tau_tc_kernel (persistent, one CTA of 608 threads per SM, one 128-row query tile at a time):
//   warp 16     TMA producer: the query tile, then the tile's key tiles through a 4-stage
//               shared-memory ring (128B-swizzled, K-major).
//   warps 17-18 issue the tcgen05.mma of S = Q K^T (M = N = 128, K = d, fp32 accumulators) into
//               one of four TMEM score buffers, so that the score warps can fall up to three
//               tiles behind during a burst of insertions; the two warps take alternate key
//               tiles (warp 17 also allocates tensor memory).  A 3-stage ring (d = 128 with the
//               larger candidate buffers) keeps one issuing warp.
//   warps 0..15 score warps: warp w reads TMEM lanes 32 (w % 4) .. + 31 (thread = query row),
//               columns 32 g .. 32 g + 31 with g = w / 4, i.e. one 32-key segment of every key
//               tile, into the segment's candidate buffer (common.cuh); the four segments of a
//               row share its running max.
//   then the score warps solve tau per row (4-lane groups), record each row's support (keys
//   with p > 0 and their p) from its candidates (record_support), and write the block mask and
//   the compact tile list.
//
// out_tc_kernel (one CTA of 384 threads per query tile, over the listed key tiles only):
//   warp 0      TMA producer of the query tile and the key tiles (3-stage ring; a key tile is
//               released as soon as its Q K^T product completes).
//   warp 2      TMA producer of the value tiles (3-stage ring, released after its P V product).
//   warp 1      tcgen05.mma: S = Q K^T into TMEM (double buffered), then O += P V with P read
//               from TMEM as the A operand and V (MN-major in shared memory) as B.
//   warps 4..11 p warps, two per TMEM lane quarter, each owning 64 keys of every tile: load S,
//               p = [c s - tau]_+^beta (0 off the causal / sequence range), store p as packed
//               bf16 into TMEM; at the end each reads half of O's columns from TMEM and stores
//               them.
// tau is known before this pass, so p needs neither a running max nor a final normalisation.
//
// Every mbarrier wait is bounded (about 2 s of %globaltimer): on expiry the waiting thread
// records ENTMAX_ATTN_ETIMEOUT in the status word and raises a CTA-wide abort flag; every role
// then leaves its loop, waits (bounded) for the copies and MMAs it issued, and the CTA frees its
// tensor memory and returns.  No trap, no unbounded spin.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace ea {
namespace {

constexpr int kOutThreads = 384;
constexpr int kScoreWarp0 = 4;            // p warps of the out pass start at warp 4 (quarter w % 4)
constexpr int kTauScoreWarps = 16;        // tau pass: warps 0..15 score, 16 TMA, 17 MMA
static_assert(kTauScoreWarps <= kXchWarps, "one exchange row per score warp");
constexpr int kTauTmaWarp = 16;
constexpr int kTauMmaWarp = 17;
constexpr int kTauThreads = 32 * (kTauScoreWarps + 2);
constexpr int kTauStages = 5;             // key tiles in flight in the tau pass
constexpr int kTauSBufs = 3;              // TMEM score buffers of the tau pass (128 columns each)
constexpr uint32_t kTauColQ = 128 * kTauSBufs;  // TMEM columns of the query tile (A operand)
constexpr uint32_t kTauTmemCols = 512;          // allocation (a power of two >= 32)
static_assert(kTauColQ + 128 / 2 <= kTauTmemCols, "score buffers + Q (d <= 128) fit in TMEM");
constexpr int kOutStages = 3;             // key tiles and value tiles in flight in the out pass

// 32 consecutive output elements from fp32 words (TMEM), at element offset e of out: rounded to
// bf16, or stored as fp32 when the caller asked for fp32 outputs (P.out_f32).  16-byte stores.
__device__ __forceinline__ void store_out32(const Problem& P, int64_t e, const uint32_t (&u)[32]) {
  if (P.out_f32) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(P.out) + e);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.out) + e);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(u[8 * i + 0]), __uint_as_float(u[8 * i + 1]));
      w.y = pack_bf16x2(__uint_as_float(u[8 * i + 2]), __uint_as_float(u[8 * i + 3]));
      w.z = pack_bf16x2(__uint_as_float(u[8 * i + 4]), __uint_as_float(u[8 * i + 5]));
      w.w = pack_bf16x2(__uint_as_float(u[8 * i + 6]), __uint_as_float(u[8 * i + 7]));
      dst[i] = w;
    }
  }
}

// n zero output elements at element offset e (n a multiple of 8).
__device__ __forceinline__ void zero_out(const Problem& P, int64_t e, int n) {
  const int bytes = n * (P.out_f32 ? 4 : 2);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(P.out) + e * (P.out_f32 ? 4 : 2));
  for (int i = 0; i < bytes / 16; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
}

// p = [x]_+^beta for the output pass, where p is rounded to bf16 before the P V product.  For
// beta = 3 + f near 3, x^beta = x^3 e^(f ln x) with the exponential cut after its linear term,
// and log2 x taken from the bits of x by Mitchell's approximation (x = 2^e (1 + m) read as
// e + m, within 0.09 of log2 x; J. N. Mitchell, "Computer multiplication and division using
// binary logarithms", 1962), so that no special-function unit is needed.  Relative error of p:
// (f ln x)^2 / 2 + |f| ln2 * 0.09 <= 5.5e-4 for x >= 1e-4 and |f| <= 0.004, below the bf16
// rounding of p (2^-9), while smaller x give p < 1e-12.  x is clamped to 1e-30 instead of 0,
// which keeps the logarithm finite and still gives p = 0 (x^3 underflows).
// With y = bits(x) >> 9 placed in the mantissa of 2^23, e + m = y 2^-14 - 639, so
// f ln x ~= y * ka + kb with ka = f ln2 2^-14 and kb = -639 f ln2.
template <int BK>
__device__ __forceinline__ float entmax_p_out(float x, float beta, float ka, float kb) {
  if (BK == kBetaNear3) {
    const float y = fmaxf(x, 1e-30f);
    const float y3 = y * y * y;
    const float e = __int_as_float((__float_as_int(y) >> 9) | 0x4B000000);
    return fmaf(y3, fmaf(e, ka, kb), y3);
  }
  return entmax_p_clamped<BK>(x, beta);
}

// p of 32 consecutive keys j0 .. j0 + 31 of a row from their raw scores (TMEM words u), packed
// as bf16 pairs; keys at or past jmax (the row's causal / sequence end) give 0.  Rows whose 32
// keys are all valid -- every tile but the diagonal one -- skip the per-key range test.
template <int BK>
__device__ __forceinline__ void p_row32(const uint32_t (&u)[32], float c, float tau, float beta,
                                        int j0, int jmax, uint32_t (&pk)[16]) {
  const float kf = (beta - 3.f) * 0.69314718f;
  const float ka = kf * (1.f / 16384.f), kb = -639.f * kf;
  if (j0 + 32 <= jmax) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = entmax_p_out<BK>(fmaf(c, __uint_as_float(u[2 * e]), -tau), beta, ka, kb);
      const float p1 = entmax_p_out<BK>(fmaf(c, __uint_as_float(u[2 * e + 1]), -tau), beta, ka, kb);
      pk[e] = pack_bf16x2(p0, p1);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 =
          (j0 + 2 * e < jmax)
              ? entmax_p_out<BK>(fmaf(c, __uint_as_float(u[2 * e]), -tau), beta, ka, kb)
              : 0.f;
      const float p1 =
          (j0 + 2 * e + 1 < jmax)
              ? entmax_p_out<BK>(fmaf(c, __uint_as_float(u[2 * e + 1]), -tau), beta, ka, kb)
              : 0.f;
      pk[e] = pack_bf16x2(p0, p1);
    }
  }
}

// ------------------------------------------------------------------------------- tau kernel --

// The tau kernel keeps Q in shared memory so that TMEM holds four 128-column score buffers: the
// score warps may fall three key tiles behind the MMA during a burst of insertions.
// Candidate slots and key stages of the tau kernel.  d = 64 leaves shared memory for 32 slots
// beside four key stages.  At d = 128, alpha other than 1.5 and 2 (the general power, e.g. 1.333)
// keeps hundreds of keys within 1 of a row's max, so its rows take 28 slots at the price of one
// key stage; alpha 1.5 and 2 keep 16 slots and four stages.
__host__ __device__ constexpr int tau_slots(int d, int bk) {
  return d == 64 ? 32 : (bk >= kBetaGeneral ? 28 : kCand);
}
__host__ __device__ constexpr int tau_stages(int d, int bk) {
  return (d == 128 && bk >= kBetaGeneral) ? 3 : 4;
}
constexpr int kMainSBufs = 4;   // TMEM score buffers

// MMA-issuing warps of the tau kernel.  A tcgen05.mma issue returns only once the tensor pipe
// has room, a few instructions deep, so a single issuing thread cannot run ahead of the pipe:
// every cycle it spends on its barrier waits and loop overhead between two groups of products
// leaves the pipe idle (clock64 counters: ~500 of ~1200 cycles per key tile).  Two warps that
// take alternate key tiles hide one's waits behind the other's issue.  Every key stage and every
// score buffer must then belong to one warp (stage and buffer counts divisible by the warp
// count), so that each warp waits on each barrier's phases in order: a warp that could wait on
// a phase two ahead of a barrier would see its parity as completed.
__host__ __device__ constexpr int tau_mma_warps(int d, int bk) {
  return (tau_stages(d, bk) % 2 == 0 && kMainSBufs % 2 == 0) ? 2 : 1;
}
__host__ __device__ constexpr int tau_threads(int d, int bk) {
  return 32 * (kTauScoreWarps + 1 + tau_mma_warps(d, bk));
}

// Query tile of a persistent CTA's round r: one tile per CTA and round, the CTAs taking them in
// reverse order every other round ("snake"), so that with the longest tiles first every CTA's
// total work comes out even (round-robin leaves the first CTAs ~3% more at 16K).
__device__ __forceinline__ int snake_tile(int r) {
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return r * g + ((r & 1) ? g - 1 - c : c);
}

// Key tiles the tau kernel visits for query tile t: every causally valid one, or with the FP8
// screen the tile's list (clamped into the tile's key range, so that no workspace content sends a
// read outside it); scr_tile gives the i-th.
__device__ __forceinline__ int scr_count(const Problem& P, const TileInfo& t) {
  return P.scr_count ? min(max(P.scr_count[t.tile_id], 0), t.nkt) : t.nkt;
}
__device__ __forceinline__ int scr_tile(const Problem& P, const TileInfo& t, int i) {
  return P.scr_list ? clamp_kt(P.scr_list[t.tile_id * P.nkt_max + i], t.nkt) : i;
}

// Steps of a query tile in the tau pass: with a warm-up level (warm_level), step 0 is the
// product with the level's 128 warm-up keys, which only raises the rows' thresholds; the key
// tiles 0 .. nkt - 1 follow in order.
__device__ __forceinline__ int warm_steps(const Problem& P, const TileInfo& t) {
  return warm_level(P, t) >= 0 ? 1 : 0;
}

template <int D, int BK>
struct TauSmem {
  static constexpr int kStages = tau_stages(D, BK);
  alignas(1024) __nv_bfloat16 q[kTile * D];
  alignas(1024) __nv_bfloat16 k[kStages][kTile * D];
  CandSmemT<tau_slots(D, BK)> cand;
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t k_full[kStages];
  uint64_t k_empty[kStages];
  uint64_t s_full[kMainSBufs];
  uint64_t s_empty[kMainSBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Every variant's shared memory (plus the 1024 bytes of alignment slack the launch adds) fits
// the 227 KB a CTA may use.
constexpr size_t kMaxSmemPerCta = 232448;
static_assert(sizeof(TauSmem<128, kBetaOne>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 128");
static_assert(sizeof(TauSmem<128, kBetaTwo>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 128");
static_assert(sizeof(TauSmem<128, kBetaGeneral>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 128");
static_assert(sizeof(TauSmem<128, kBetaNear3>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 128");
static_assert(sizeof(TauSmem<64, kBetaGeneral>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 64");
static_assert(sizeof(TauSmem<64, kBetaNear3>) + 1024 <= kMaxSmemPerCta, "tau smem, d = 64");

// Score warps only (named barrier 1): a barrier, and a barrier that also returns whether any
// score thread passed a true flag (the same answer in every thread).
__device__ __forceinline__ void score_warps_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kTauScoreWarps) : "memory");
}
__device__ __forceinline__ bool score_warps_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n"
      " barrier.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"(static_cast<int>(flag)), "n"(32 * kTauScoreWarps)
      : "memory");
  return r != 0;
}

// Supports from the candidates.  Every key with p_ij > 0 has z_ij > tau_i >= m_i - 1, so once a
// row's candidate buffers hold every key above their floor and tau lies above the floor (what
// solve_rows checks; a tile that fails is queued for the overflow path), the row's support is
// exactly its buffer entries with z > tau.  The support of a row is a handful of keys where the
// tile output pass would multiply whole 128-key tiles of mostly zero p; so the tau kernel records
// each row's support -- key j of the sequence and p_ij in fp32 from the stored raw score and tau
// -- in its query tile's list (rows one after another, kSupPerTile entries per tile), and the
// output pass computes o_i = sum p_ij v_j from the lists (out_support_kernel).  A tile whose rows
// need more entries than its list holds is left pending for the tile output pass.  Call from all
// score threads (one row per 4-lane group) after the barrier that follows solve_rows; it holds
// two barriers of the score warps.
template <int BK, class CS>
__device__ __forceinline__ void record_support(const Problem& P, const TileInfo& t, CS& cs,
                                               int tid, int lane) {
  const unsigned full = 0xffffffffu;
  const int lane4 = tid & 3;
  const int r = tid >> 2;  // 512 score threads: one row per 4-lane group
  const bool valid = r < t.nrows;
  const float tau = valid ? cs.tau_r[r] : 0.f;
  // This lane's share of the row's entries: e = lane4 + 4 i of every segment g, bit
  // g * kPer + i of take when the entry lies in the support.  The test is made once and the
  // writes below follow the bits: evaluated twice, z - tau of a key within rounding of tau could
  // come out on different sides (the compiler may fuse the product and the difference in one place
  // and not in the other), and the row would write one entry more or less than it counted, into
  // the next row's part of the list.  z - tau is rounded step by step (no fused multiply-add), so
  // the value the writes recompute is the one tested.
  constexpr int kPer = CS::kSlots / 4;
  static_assert(kSeg * kPer <= 32, "one bit per entry of a lane's share");
  uint32_t take = 0u;
  if (valid) {
#pragma unroll 1
    for (int g = 0; g < kSeg; ++g) {
      const int col = g * kTile + r;
      const int cnt = min(cs.cnt[col], CS::kSlots);
      for (int e = lane4, i = 0; e < cnt; e += 4, ++i)
        if (__fsub_rn(__fmul_rn(P.c, cs.s[e * kCols + col]), tau) > 0.f)
          take |= 1u << (g * kPer + i);
    }
  }
  const int n = __popc(take);
  // the row's total and this lane's first entry among the row's four lanes
  int incl = n;
  int y = __shfl_up_sync(full, incl, 1);
  if (lane4 >= 1) incl += y;
  y = __shfl_up_sync(full, incl, 2);
  if (lane4 >= 2) incl += y;
  const int total = __shfl_sync(full, incl, (lane & ~3) | 3);
  if (lane4 == 3) cs.sup_n[r] = total;
  score_warps_sync();
  if (tid < 32) {  // exclusive prefix over the 128 rows: four rows per lane
    int a[4], sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = sum;
      sum += cs.sup_n[4 * tid + i];
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int z = __shfl_up_sync(full, x, o);
      if (tid >= o) x += z;
    }
    const int base = x - sum;
#pragma unroll
    for (int i = 0; i < 4; ++i) cs.sup_n[4 * tid + i] = base + a[i];
    if (tid == 31) cs.sup_over = x > kSupPerTile ? 1 : 0;
  }
  score_warps_sync();
  if (cs.sup_over || !valid) return;
  int2* list = P.sup + t.tile_id * kSupPerTile;
  const int first = cs.sup_n[r];
  int at = first + incl - n;
#pragma unroll 1
  for (int g = 0; g < kSeg; ++g) {
    const int col = g * kTile + r;
    const int cnt = min(cs.cnt[col], CS::kSlots);
    for (int e = lane4, i = 0; e < cnt; e += 4, ++i) {
      if ((take >> (g * kPer + i)) & 1u) {
        const float x = __fsub_rn(__fmul_rn(P.c, cs.s[e * kCols + col]), tau);  // > 0, as tested
        const int id = cs.kt[e * kCols + col];
        const int j = (id >> 5) * kTile + g * 32 + (id & 31);  // key of the sequence
        list[at++] = make_int2(j, __float_as_int(entmax_p<BK>(x, P.beta)));
      }
    }
  }
  if (lane4 == 0) P.sup_idx[t.qhead + t.seq_start + t.row0 + r] = first | (total << 16);
}

template <int D, int BK>
__global__ void __launch_bounds__(tau_threads(D, BK), 1)
    tau_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmw, Problem P) {
  constexpr int kStages = TauSmem<D, BK>::kStages;
  constexpr int kMmaWarps = tau_mma_warps(D, BK);
  constexpr int kThreads = tau_threads(D, BK);
  static_assert(kStages % kMmaWarps == 0 && kMainSBufs % kMmaWarps == 0,
                "each key stage and score buffer belongs to one MMA warp");
  extern __shared__ unsigned char smem_raw[];
  TauSmem<D, BK>& sm = *reinterpret_cast<TauSmem<D, BK>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto& cs = sm.cand;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int per_slot = P.Hq * (P.cu ? 1 : P.B);
  const int ntiles = P.slots * per_slot;
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * D * 2;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, kMmaWarps);  // one commit per MMA warp
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int b = 0; b < kMainSBufs; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_empty[b], kTauScoreWarps);  // one arrival per score warp
    }
    mbar_init(&sm.drain, kMmaWarps);
    sm.abort = 0;
    cs.fallback = P.force_fallback;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int w = tid; w < kMaxWords; w += kThreads) cs.words[w] = 0u;
  if (warp == kTauMmaWarp) tmem_alloc(&sm.tmem_base, kTauTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Every role walks the same tiles L = blockIdx.x, blockIdx.x + gridDim.x, ...; the rings
  // (key stages, score buffers) and the query buffer's phases run on across tiles, so the
  // producer and the MMA thread start on the next tile while the score warps finish this one.
  if (warp == kTauTmaWarp) {
    if (lane == 0) {
      int it = 0, gk = 0;  // tiles and key tiles issued so far
      bool ok = true;
      int rr = 0;
      for (int L = snake_tile(0); ok && L < ntiles; L = snake_tile(++rr)) {
        const TileInfo t = tau_tile(P, L, per_slot);
        if (!t.valid) continue;
        // the query buffer is free once every S product of the previous tile has completed
        if (it > 0 && !mbar_wait(&sm.q_empty, (it - 1) & 1, abort, P.status)) break;
        const int qrow = static_cast<int>(t.qhead + t.seq_start + t.row0);
        const int krow0 = static_cast<int>(t.khead + t.seq_start);
        if (!P.test_stall) {  // the test hook leaves q_full incomplete: every wait runs out
          mbar_expect_tx(&sm.q_full, kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_2d(sm.q + h * kTile * 64, &tmq, &sm.q_full, h * 64, qrow);
        }
        // the query tile this CTA takes next comes from HBM: start it towards L2 now, so that its
        // load, issued only once this tile's products are done, finds it there
        if (snake_tile(rr + 1) < ntiles) {
          const TileInfo tn = tau_tile(P, snake_tile(rr + 1), per_slot);
          if (tn.valid)
            for (int h = 0; h < D / 64; ++h)
              tma_prefetch_2d(&tmq, h * 64, static_cast<int>(tn.qhead + tn.seq_start + tn.row0));
        }
        ++it;
        const int lvl = warm_level(P, t), ws = lvl >= 0 ? 1 : 0, nsteps = scr_count(P, t) + ws;
        const int wrow = (t.grp * P.warm_levels + lvl) * kTile;
        for (int i = 0; i < nsteps; ++i, ++gk) {
          const int s = gk % kStages;
          if (gk >= kStages &&
              !mbar_wait(&sm.k_empty[s], ((gk / kStages) - 1) & 1, abort, P.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&sm.k_full[s], kTileBytes);
          if (i < ws) {
            for (int h = 0; h < D / 64; ++h)
              tma_load_2d(sm.k[s] + h * kTile * 64, &tmw, &sm.k_full[s], h * 64, wrow);
          } else {
            const int kt = scr_tile(P, t, i - ws);
            for (int h = 0; h < D / 64; ++h)
              tma_load_2d(sm.k[s] + h * kTile * 64, &tmk, &sm.k_full[s], h * 64,
                          krow0 + kt * kTile);
          }
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int g = (gk > kStages ? gk - kStages : 0); g < gk; ++g)
        mbar_wait(&sm.k_full[g % kStages], (g / kStages) & 1, abort, P.status);
      if (it > 0) mbar_wait(&sm.q_full, (it - 1) & 1, abort, P.status);
    }
  } else if (warp >= kTauMmaWarp) {
    if (lane == 0) {
      const int mine = warp - kTauMmaWarp;  // this warp issues the groups gk % kMmaWarps == mine
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
      uint64_t qdesc[D / 16];
#pragma unroll
      for (int k16 = 0; k16 < D / 16; ++k16) qdesc[k16] = kmajor_desc(smem_u32(sm.q), kTile, k16);
      const uint64_t kdesc0 = kmajor_desc(smem_u32(sm.k[0]), kTile, 0);
      int it = 0, gk = 0;  // tiles and key tiles consumed so far (one S buffer per key tile)
      bool ok = true;
      int rr = 0;
      for (int L = snake_tile(0); ok && L < ntiles; L = snake_tile(++rr)) {
        const TileInfo t = tau_tile(P, L, per_slot);
        if (!t.valid) continue;
        if (!mbar_wait(&sm.q_full, it & 1, abort, P.status)) break;
        ++it;
        const int nsteps = scr_count(P, t) + warm_steps(P, t);
        for (int i = 0; i < nsteps; ++i, ++gk) {
          if (gk % kMmaWarps != mine) continue;
          const int s = gk % kStages, b = gk % kMainSBufs;
          if (!mbar_wait(&sm.k_full[s], (gk / kStages) & 1, abort, P.status) ||
              (gk >= kMainSBufs &&
               !mbar_wait(&sm.s_empty[b], ((gk / kMainSBufs) - 1) & 1, abort, P.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = desc_add(kdesc0, static_cast<uint32_t>(s) * kTileBytes);
          const uint32_t dcol = tmem + static_cast<uint32_t>(b * 128);
#pragma unroll
          for (int k16 = 0; k16 < D / 16; ++k16)
            mma_ss(dcol, qdesc[k16],
                   desc_add(kd, static_cast<uint32_t>((k16 >> 2) * kTile * 128 + (k16 & 3) * 32)),
                   idesc, k16 > 0 ? 1u : 0u);
          mma_commit(&sm.k_empty[s]);
          mma_commit(&sm.s_full[b]);
        }
        if (ok) mma_commit(&sm.q_empty);  // this warp's S products of the tile have read Q
      }
      if (gk > 0) {  // all issued MMAs complete before tensor memory is released
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, abort, P.status);
      }
    }
  } else {  // score warps 0..15
    const int quarter = warp & 3;
    const int seg = warp >> 2;  // keys 32 seg .. 32 seg + 31 of every key tile
    const int r = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const int col = seg * kTile + r;
    constexpr int kScoreThreads = 32 * kTauScoreWarps;
    int gs = 0;  // score buffers consumed so far
    int rr = 0;
    for (int L = snake_tile(0); L < ntiles; L = snake_tile(++rr)) {
      const TileInfo t = tau_tile(P, L, per_slot);
      if (!t.valid) {
        emit_empty(P, t, tid, kScoreThreads);
        continue;
      }
      // per-tile shared state: the row max now; the mask words and the overflow flag, which the
      // previous tile's emit read, once every score thread has passed the barrier below
      if (tid < kTile) cs.rowmax[tid] = -INFINITY;  // warps 0..3: thread tid owns row tid
      score_warps_sync();
      if (tid < kMaxWords) cs.words[tid] = 0u;
      if (tid == 0) cs.fallback = P.force_fallback;
      const int ws = warm_steps(P, t), nsteps = scr_count(P, t) + ws;
      const int jmax = (r < t.nrows) ? (P.causal ? t.row0 + r + 1 : t.seq_len) : 0;
      RowCand rc;
      rc.init(1.f / P.c);
      for (int i = 0; i < nsteps; ++i, ++gs) {
        const int b = gs % kMainSBufs;
        const int kt = i < ws ? -1 : scr_tile(P, t, i - ws);  // -1: the warm-up keys
        // the warp leaves together: feed_warp needs all 32 lanes
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&sm.s_full[b], (gs / kMainSBufs) & 1, abort, P.status)))
          break;
        tc_fence_after();
        const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(b * 128 + seg * 32);
        float x[32];
        if (kt < 0)  // every warm-up key is visible to every row of the tile
          tmem_row32(ta, 0, r < t.nrows ? kTile : 0, x);
        else
          tmem_row32(ta, kt * kTile + seg * 32, jmax, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_empty[b]);  // scores are in registers: release S[b]
        if (kt < 0)
          observe_bound(rc, cs, r, x);
        else
          feed_warp<32>(rc, cs, cs.xrow[warp], col, r, lane, x, kt);
      }
      rc.publish(cs, col);
      if (score_warps_any(*abort != 0)) break;  // status already records the timeout
      solve_rows<BK>(P, t, cs, tid, kScoreThreads);
      score_warps_sync();
      if (P.record_support) {  // unless the tile goes to the overflow path (uniform test)
        if (!cs.fallback) record_support<BK>(P, t, cs, tid, lane);
        if (tid == 0) P.pending[t.tile_id] = (cs.fallback || cs.sup_over) ? 1 : 0;
      }
      if (warp == 0) emit_tile_prefix(P, t, cs, lane);
      score_warps_sync();
      emit_tile_entries(P, t, cs, tid, kScoreThreads);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTauMmaWarp) tmem_dealloc(tmem, kTauTmemCols);
}

// ---------------------------------------------------------------------- tau overflow kernel --
// tau_tc_sweep_kernel: the exact tau search for query tiles whose candidate buffers overflowed,
// with no candidate buffers at all.  S = Q K^T is recomputed on the tensor cores for every sweep
// over the tile's key range: one sweep for the row max, one per search step (the sums of
// (z - tau)^beta, ^(beta - 1), ^(beta - 2) over all keys with z > tau), one for the mask bits
// and, with the supports recorded, one for the support lists.  Roles as in tau_tc_kernel; the
// four segment threads of a row combine their partial results through shared memory after every
// sweep.  CTAs loop over the overflow queue.

template <int D>
struct SweepSmem {
  alignas(1024) __nv_bfloat16 k[kTauStages][kTile * D];
  float part[2][3][kSeg][kTile];  // per-sweep partials, double-buffered by sweep parity
  uint32_t words[kMaxWords];
  int sup_cnt[kSeg][kTile];  // support entries of each (segment, row), counted by the mask round
  int sup_first[kTile];      // the row's first position in the tile's support list
  int sup_total[kTile];
  int sup_over;              // the tile's supports do not fit its list
  uint64_t q_full;
  uint64_t k_full[kTauStages];
  uint64_t k_empty[kTauStages];
  uint64_t s_full[kTauSBufs];
  uint64_t s_empty[kTauSBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int kind;  // what the current round over the tile does (row max, search step, mask bits,
             // support entries)
};

template <int D, int BK>
__global__ void __launch_bounds__(kTauThreads, 1)
    tau_tc_sweep_kernel(const __grid_constant__ CUtensorMap tmk, Problem P) {
  extern __shared__ unsigned char smem_raw[];
  SweepSmem<D>& sm = *reinterpret_cast<SweepSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int ntiles = (P.cu ? 1 : P.B) * P.Hq * P.slots;
  const int nq = min(*P.queue_count, ntiles);
  if (static_cast<int>(blockIdx.x) >= nq) return;  // nothing queued for this CTA
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  const unsigned full = 0xffffffffu;

  if (tid == 0) {
    mbar_init(&sm.q_full, kTauScoreWarps);
    for (int s = 0; s < kTauStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int b = 0; b < kTauSBufs; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_empty[b], kTauScoreWarps);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    sm.kind = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int w = tid; w < kMaxWords; w += kTauThreads) sm.words[w] = 0u;
  if (warp == kTauMmaWarp) tmem_alloc(&sm.tmem_base, kTauTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  int g = 0;       // key-tile steps so far in this CTA (identical in every role)
  int tcount = 0;  // tiles so far (phase of q_full)
  int issued_total = 0;

  for (int i = blockIdx.x; i < nq; i += gridDim.x) {
    const int id = P.queue[i];
    if (id < 0 || id >= ntiles) continue;  // uniform across the block
    const TileInfo t = map_tile(P, id % P.slots, (id / P.slots) % P.Hq, id / (P.slots * P.Hq));
    const int nkt = t.nkt;
    const int quarter = warp & 3;
    const int seg = warp >> 2;
    const int r = quarter * 32 + lane;
    const bool valid = r < t.nrows;
    const int jmax = valid ? (P.causal ? t.row0 + r + 1 : t.seq_len) : 0;
    Search sr;  // score warps: the row's search
    int steps_done = 0;
    if (warp < kTauScoreWarps) {  // this thread's quarter of its query row into TMEM
      constexpr int kWords = D / 8;
      uint32_t w[kWords];
      if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(P.q) + (t.qhead + t.seq_start + t.row0 + r) * D +
            seg * (D / 4));
#pragma unroll
        for (int e = 0; e < kWords / 4; ++e) {
          const uint4 u = src[e];
          w[4 * e] = u.x;
          w[4 * e + 1] = u.y;
          w[4 * e + 2] = u.z;
          w[4 * e + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < kWords; ++e) w[e] = 0u;
      }
      tmem_st_words<kWords>(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kTauColQ +
                                static_cast<uint32_t>(seg * kWords),
                            w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
      sr.init(0.f, 1, P.alpha);
    }
    // One sweep of S over the tile's key range per round; what a round does (row max, one
    // search step, mask bits, support entries) is decided by the score warps at the end of the
    // round before and published in sm.kind behind a CTA barrier, so that every role runs the
    // same rounds.  The search stops as soon as every row of the tile has settled (at most
    // n_iter steps).  With the supports recorded (P.record_support), the mask round also counts
    // each row's keys with z > tau, and when the tile's rows fit its list one more round writes
    // them there (key and p, as the main kernel's record_support does): the tile then leaves the
    // pending set and its output and gradients come from the lists as well.  Both rounds test
    // z - tau rounded step by step on the same products, so that they agree key by key.
    int sup_at = 0, sup_left = 0;  // score threads: this (row, segment)'s next entry and quota
    bool sup_done = false;
    for (;;) {
      const int kind = sm.kind;  // 0 row max, 1 search step, 2 mask bits, 4 support entries
      if (warp == kTauTmaWarp) {
        if (lane == 0) {
          const int krow0 = static_cast<int>(t.khead + t.seq_start);
          for (int kt = 0; kt < nkt; ++kt) {
            const int gg = g + kt, s = gg % kTauStages;
            if (gg >= kTauStages &&
                !mbar_wait(&sm.k_empty[s], ((gg / kTauStages) - 1) & 1, abort, P.status))
              break;
            mbar_expect_tx(&sm.k_full[s], kTileBytes);
            for (int h = 0; h < D / 64; ++h)
              tma_load_2d(sm.k[s] + h * kTile * 64, &tmk, &sm.k_full[s], h * 64,
                          krow0 + kt * kTile);
            issued_total = gg + 1;
          }
        }
      } else if (warp == kTauMmaWarp) {
        if (lane == 0) {
          constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
          bool ok = kind != 0 || mbar_wait(&sm.q_full, tcount & 1, abort, P.status);
          for (int kt = 0; ok && kt < nkt; ++kt) {
            const int gg = g + kt, s = gg % kTauStages, b = gg % kTauSBufs;
            if (!mbar_wait(&sm.k_full[s], (gg / kTauStages) & 1, abort, P.status)) break;
            if (gg >= kTauSBufs &&
                !mbar_wait(&sm.s_empty[b], ((gg / kTauSBufs) - 1) & 1, abort, P.status))
              break;
            tc_fence_after();
            const uint32_t kbase = smem_u32(sm.k[s]);
#pragma unroll
            for (int k16 = 0; k16 < D / 16; ++k16)
              mma_ts(tmem + static_cast<uint32_t>(b * 128), tmem + kTauColQ + k16 * 8,
                     kmajor_desc(kbase, kTile, k16), idesc, k16 > 0 ? 1u : 0u);
            mma_commit(&sm.k_empty[s]);
            mma_commit(&sm.s_full[b]);
            issued_total = gg + 1;
          }
        }
      } else {  // score warps 0..15: every step of the round, even after an abort (barriers)
        float a0 = (kind == 0) ? -INFINITY : 0.f, a1 = 0.f, a2 = 0.f;
        const float tau = sr.tau;
        for (int kt = 0; kt < nkt; ++kt) {
          const int gg = g + kt, b = gg % kTauSBufs;
          const bool okw = __all_sync(
              full, !*abort && mbar_wait(&sm.s_full[b], (gg / kTauSBufs) & 1, abort, P.status));
          if (!okw) continue;
          tc_fence_after();
          float x[32];
          tmem_row32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                         static_cast<uint32_t>(b * 128 + seg * 32),
                     kt * kTile + seg * 32, jmax, x);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_empty[b]);
          if (kind == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) a0 = fmaxf(a0, x[e]);
          } else if (kind == 1) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float y = P.c * x[e] - tau;
              if (y > 0.f) {
                float p0, p1, p2;
                entmax_powers<BK>(y, P.beta, p0, p1, p2);
                a0 += p0;
                a1 += p1;
                a2 += p2;
              }
            }
          } else if (kind == 2) {
            int n = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) n += (__fsub_rn(__fmul_rn(P.c, x[e]), tau) > 0.f) ? 1 : 0;
            if (n) atomicOr(&sm.words[kt >> 5], 1u << (kt & 31));
            a0 += static_cast<float>(n);  // exact: at most 32 per key tile, 2^24 in all
          } else if (sup_left > 0) {  // kind 4: this (row, segment)'s entries, in key order
            int2* list = P.sup + t.tile_id * kSupPerTile;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float y = __fsub_rn(__fmul_rn(P.c, x[e]), tau);
              if (y > 0.f && sup_left > 0) {
                list[sup_at++] = make_int2(kt * kTile + seg * 32 + e,
                                           __float_as_int(entmax_p<BK>(y, P.beta)));
                --sup_left;
              }
            }
          }
        }
        int next = 3;  // done
        if (kind == 2 && P.record_support) {
          // the rows' places in the tile's list: segments one after another within a row, rows
          // one after another; the tile keeps its pending flag if they do not fit
          sm.sup_cnt[seg][r] = valid ? static_cast<int>(a0) : 0;
          score_warps_sync();
          if (tid < 32) {  // exclusive prefix over the 128 rows: four rows per lane
            int a[4], sum = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = 4 * tid + i;
              const int n = sm.sup_cnt[0][row] + sm.sup_cnt[1][row] + sm.sup_cnt[2][row] +
                            sm.sup_cnt[3][row];
              sm.sup_total[row] = n;
              a[i] = sum;
              sum += n;
            }
            int x = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int z = __shfl_up_sync(full, x, o);
              if (tid >= o) x += z;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) sm.sup_first[4 * tid + i] = x - sum + a[i];
            if (tid == 31) sm.sup_over = x > kSupPerTile ? 1 : 0;
          }
          score_warps_sync();
          sup_at = sm.sup_first[r];
#pragma unroll
          for (int q2 = 0; q2 < kSeg; ++q2) sup_at += (q2 < seg) ? sm.sup_cnt[q2][r] : 0;
          sup_left = sm.sup_cnt[seg][r];
          if (!sm.sup_over) next = 4;
        } else if (kind == 4) {
          // the entries a row counted but did not find again (none while the tensor cores
          // return the same products for the same operands) are left as p = 0 at key 0
          int2* list = P.sup + t.tile_id * kSupPerTile;
          for (; sup_left > 0; --sup_left) list[sup_at++] = make_int2(0, 0);
          sup_done = true;
        }
        if (kind != 2 && kind != 4) {
          const int pb = steps_done & 1;
          sm.part[pb][0][seg][r] = a0;
          sm.part[pb][1][seg][r] = a1;
          sm.part[pb][2][seg][r] = a2;
          score_warps_sync();
          float t0 = sm.part[pb][0][0][r], t1 = sm.part[pb][1][0][r], t2 = sm.part[pb][2][0][r];
#pragma unroll
          for (int q2 = 1; q2 < kSeg; ++q2) {
            if (kind == 0) {
              t0 = fmaxf(t0, sm.part[pb][0][q2][r]);
            } else {
              t0 += sm.part[pb][0][q2][r];
              t1 += sm.part[pb][1][q2][r];
              t2 += sm.part[pb][2][q2][r];
            }
          }
          if (kind == 0) {
            sr.init(valid ? P.c * t0 : 0.f, valid ? jmax : 1, P.alpha);
            // start from the tau the main pass found on the candidates it kept: a lower bound
            // of the row's tau when finite, and inside the bracket either way
            const float t_kept = valid ? P.tau[t.qhead + t.seq_start + t.row0 + r] : sr.lo;
            if (t_kept > sr.lo && t_kept < sr.hi) sr.tau = t_kept;
            next = 1;
          } else {
            sr.step<BK>(t0, t1, t2, P.beta);
            ++steps_done;
            const bool busy = valid && !sr.settled();
            next = (steps_done < P.n_iter && score_warps_any(busy)) ? 1 : 2;
          }
        }
        if (*abort) next = 3;
        score_warps_sync();  // every score thread has read sm.kind of this round
        if (tid == 0) sm.kind = next;
      }
      g += nkt;
      tc_fence_before();
      __syncthreads();  // the next round's kind is published
      tc_fence_after();
      if (sm.kind == 3) break;
    }
    if (warp < kTauScoreWarps && seg == 0 && valid) {
      const int64_t row = t.qhead + t.seq_start + t.row0 + r;
      P.tau[row] = sr.tau;
      if (sup_done) P.sup_idx[row] = sm.sup_first[r] | (sm.sup_total[r] << 16);
    }
    // the tile's lists are complete: it leaves the pending set (the output pass runs after)
    if (tid == 0 && sup_done && !*abort) P.pending[t.tile_id] = 0;
    ++tcount;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!*abort && warp == 0) emit_tile(P, t, sm.words, 0, lane);
    __syncthreads();
    for (int w = tid; w < kMaxWords; w += kTauThreads) sm.words[w] = 0u;
    if (tid == 0) sm.kind = 0;
    __syncthreads();
  }
  // drain: issued copies have landed and issued MMAs have completed before TMEM is released
  if (warp == kTauTmaWarp && lane == 0) {
    for (int gg = (issued_total > kTauStages ? issued_total - kTauStages : 0); gg < issued_total;
         ++gg)
      mbar_wait(&sm.k_full[gg % kTauStages], (gg / kTauStages) & 1, abort, P.status);
  }
  if (warp == kTauMmaWarp && lane == 0 && issued_total > 0) {
    mma_commit(&sm.drain);
    mbar_wait(&sm.drain, 0, abort, P.status);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTauMmaWarp) tmem_dealloc(tmem, kTauTmemCols);
}

// ------------------------------------------------------------------------------- out kernel --

template <int D>
struct OutSmem {
  alignas(1024) __nv_bfloat16 q[kTile * D];
  alignas(1024) __nv_bfloat16 k[kOutStages][kTile * D];
  alignas(1024) __nv_bfloat16 v[kOutStages][kTile * D];
  uint64_t q_full;
  uint64_t k_full[kOutStages];
  uint64_t k_empty[kOutStages];
  uint64_t v_full[kOutStages];
  uint64_t v_empty[kOutStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t p_free[2];  // PV MMA that read P[b] has completed
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
};

// TMEM columns: S[0], S[1] at 0 and 128; P[0], P[1] (128 keys as 64 packed bf16x2 columns) at
// 256 and 320; O (d fp32 columns) at 384.
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;

template <int D, int BK>
__global__ void __launch_bounds__(kOutThreads, 1)
    out_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, Problem P) {
  extern __shared__ unsigned char smem_raw[];
  OutSmem<D>& sm = *reinterpret_cast<OutSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int slot = gridDim.x - 1 - blockIdx.x;
  const TileInfo t = map_tile(P, slot, blockIdx.y, blockIdx.z);
  if (!t.valid) return;
  if (P.from_support && P.pending[t.tile_id] == 0) return;  // o from the tile's support list
  // The list comes from the tau pass; clamping keeps every read inside this tile's list and key
  // range even if the workspace was never filled.
  const int cnt = list_count(P, t);
  const int* list = P.list + t.tile_id * P.nkt_max;
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * D * 2;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kOutStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], 8);  // one arrival per p warp
      mbar_init(&sm.p_free[b], 1);
    }
    mbar_init(&sm.o_full, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // warp 0 streams Q and the key tiles, warp 2 the value tiles
      const bool keys = warp == 0;
      const CUtensorMap* map = keys ? &tmk : &tmv;
      __nv_bfloat16(*ring)[kTile * D] = keys ? sm.k : sm.v;
      uint64_t* full = keys ? sm.k_full : sm.v_full;
      uint64_t* empty = keys ? sm.k_empty : sm.v_empty;
      const int krow0 = static_cast<int>(t.khead + t.seq_start);
      if (keys) {
        const int qrow = static_cast<int>(t.qhead + t.seq_start + t.row0);
        mbar_expect_tx(&sm.q_full, kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d(sm.q + h * kTile * 64, &tmq, &sm.q_full, h * 64, qrow);
      }
      int issued = 0;
      for (int i = 0; i < cnt; ++i) {
        const int s = i % kOutStages;
        if (i >= kOutStages &&
            !mbar_wait(&empty[s], ((i / kOutStages) - 1) & 1, abort, P.status))
          break;
        const int row = krow0 + list_tile(P, list, i, t.nkt) * kTile;
        mbar_expect_tx(&full[s], kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d(ring[s] + h * kTile * 64, map, &full[s], h * 64, row);
        issued = i + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int i = (issued > kOutStages ? issued - kOutStages : 0); i < issued; ++i)
        mbar_wait(&full[i % kOutStages], (i / kOutStages) & 1, abort, P.status);
      if (keys) mbar_wait(&sm.q_full, 0, abort, P.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);
      const uint32_t qbase = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.q_full, 0, abort, P.status);
      // S(i) = Q K(i)^T into S[i & 1]
      auto issue_s = [&](int i) -> bool {
        const int s = i % kOutStages, b = i & 1;
        if (!mbar_wait(&sm.k_full[s], (i / kOutStages) & 1, abort, P.status)) return false;
        // S[b] is free once the p warps have read S(i-2): they signal that through p_full.
        if (i >= 2 && !mbar_wait(&sm.p_full[b], ((i >> 1) - 1) & 1, abort, P.status))
          return false;
        tc_fence_after();
        const uint32_t kbase = smem_u32(sm.k[s]);
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16)
          mma_ss(tmem + kColS + b * 128, kmajor_desc(qbase, kTile, k16),
                 kmajor_desc(kbase, kTile, k16), idesc_s, k16 > 0 ? 1u : 0u);
        mma_commit(&sm.k_empty[s]);
        mma_commit(&sm.s_full[b]);
        return true;
      };
      int done = 0;  // PV products issued
      if (ok && cnt > 0) ok = issue_s(0);
      for (int i = 0; ok && i < cnt; ++i) {
        const int s = i % kOutStages, b = i & 1;
        if (i + 1 < cnt && !issue_s(i + 1)) break;
        if (!mbar_wait(&sm.p_full[b], (i >> 1) & 1, abort, P.status)) break;
        if (!mbar_wait(&sm.v_full[s], (i / kOutStages) & 1, abort, P.status)) break;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sm.v[s]);
#pragma unroll
        for (int k16 = 0; k16 < kTile / 16; ++k16)
          mma_ts(tmem + kColO, tmem + kColP + b * 64 + k16 * 8, value_desc(vbase, k16), idesc_o,
                 (i > 0 || k16 > 0) ? 1u : 0u);
        mma_commit(&sm.v_empty[s]);
        mma_commit(&sm.p_free[b]);
        done = i + 1;
      }
      (void)done;
      mma_commit(&sm.o_full);  // arrives once every MMA issued so far has completed
    }
  } else if (warp >= kScoreWarp0) {
    const int quarter = warp & 3;
    const int half = (warp - kScoreWarp0) >> 2;  // keys 64 half .. 64 half + 63 of every tile
    const int r = quarter * 32 + lane;
    const bool row_ok = r < t.nrows;
    const int pos = t.row0 + r;
    const int jmax = row_ok ? (P.causal ? pos + 1 : t.seq_len) : 0;
    const float tau = row_ok ? P.tau[t.qhead + t.seq_start + pos] : INFINITY;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    for (int i = 0; i < cnt; ++i) {
      const int b = i & 1;
      const int kt = list_tile(P, list, i, t.nkt);
      if (!mbar_wait(&sm.s_full[b], (i >> 1) & 1, abort, P.status)) break;
      // P[b] is free once the PV product of step i-2 has completed
      if (i >= 2 && !mbar_wait(&sm.p_free[b], ((i >> 1) - 1) & 1, abort, P.status)) break;
      tc_fence_after();
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int c0 = half * 64 + q2 * 32;  // S column == key offset in the tile
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + kColS + b * 128 + c0, u);
        uint32_t pk[16];
        p_row32<BK>(u, P.c, tau, P.beta, kt * kTile + c0, jmax, pk);
        tmem_st16(tmem + lane_off + kColP + b * 64 + c0 / 2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[b]);
    }
    // epilogue: this warp's half of O's columns, from TMEM to global memory
    const bool o_ok = mbar_wait(&sm.o_full, 0, abort, P.status);
    tc_fence_after();
    constexpr int kHalfD = D / 2;
    const int64_t oe = (t.qhead + t.seq_start + pos) * D + half * kHalfD;  // element offset
    if (o_ok && !*abort && cnt == 0 && row_ok) {  // no listed tile (only after a failed tau pass)
      zero_out(P, oe, kHalfD);
    } else if (o_ok && !*abort) {
#pragma unroll 1
      for (int c0 = 0; c0 < kHalfD; c0 += 32) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + kColO + half * kHalfD + c0, u);
        if (row_ok) store_out32(P, oe + c0, u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------- paired-head out kernel --
// out_pair_kernel: the output pass for two query heads of one GQA group (same key/value head,
// same query tile), so that every key and value tile is loaded once for both.  The tile walks
// the union of the two heads' compact lists; each head computes S and O only on its own listed
// tiles.  TMEM holds S_A, S_B (128 columns each) and O_A, O_B; P is written back over the S
// columns its warp has already read (keys 64 h + 32 q of the tile -> columns 64 h + 16 q), so
// the PV product of head X on a tile and the next S of head X are issued back to back and the
// tensor pipe always holds the other head's work while one head's p warps run:
//   ... PV_A(u), S_A(u+1), PV_B(u), S_B(u+1), PV_A(u+1), ...
// tcgen05.mma instructions of a CTA execute in issue order, so S_X(u+1) overwrites the columns
// PV_X(u) reads only after PV_X(u) has read them.
//   warp 0       TMA producer of both query tiles and the key tiles (kPairKStages-stage ring)
//   warp 1       tcgen05.mma issue (one thread)
//   warp 2       TMA producer of the value tiles (kPairVStages-stage ring)
//   warps 4..11  p warps of head A, warps 12..19 of head B (quarter w % 4, 64-key half)
constexpr int kPairThreads = 640;
constexpr int kPairKStages = 3;
constexpr int kPairVStages = 2;
constexpr uint32_t kPairColO = 256;  // O_A at 256, O_B at 384 (d <= 128 columns each)

template <int D>
struct PairSmem {
  alignas(1024) __nv_bfloat16 q[2][kTile * D];
  alignas(1024) __nv_bfloat16 k[kPairKStages][kTile * D];
  alignas(1024) __nv_bfloat16 v[kPairVStages][kTile * D];
  uint64_t q_full;
  uint64_t k_full[kPairKStages];
  uint64_t k_empty[kPairKStages];
  uint64_t v_full[kPairVStages];
  uint64_t v_empty[kPairVStages];
  uint64_t s_full[2];  // per head: S_X of its next listed tile is in TMEM
  uint64_t p_full[2];  // per head: its p warps have read S_X and stored P_X (8 arrivals)
  uint64_t o_full;
  uint32_t tmem_base;
  int abort;
};

// Merged walk over two ascending compact lists (entries clamped to the tile's key range): each
// step yields the next key tile and whether either list holds it.  Advances at least one list
// per step, so it ends after at most na + nb steps whatever the lists hold.
struct UnionWalk {
  const int* la;
  const int* lb;
  int na, nb, ia, ib, nkt;
  int all;  // no block mask: both lists are 0, 1, ..., nkt - 1
  __device__ __forceinline__ bool next(int& kt, bool& in_a, bool& in_b) {
    if (ia >= na && ib >= nb) return false;
    const int a = ia < na ? (all ? ia : clamp_kt(la[ia], nkt)) : INT_MAX;
    const int b = ib < nb ? (all ? ib : clamp_kt(lb[ib], nkt)) : INT_MAX;
    kt = min(a, b);
    in_a = a == kt;
    in_b = b == kt;
    ia += in_a ? 1 : 0;
    ib += in_b ? 1 : 0;
    return true;
  }
};

template <int D, int BK>
__global__ void __launch_bounds__(kPairThreads, 1)
    out_pair_kernel(const __grid_constant__ CUtensorMap tmq,
                    const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmo, Problem P) {
  extern __shared__ unsigned char smem_raw[];
  PairSmem<D>& sm = *reinterpret_cast<PairSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int slot = gridDim.x - 1 - blockIdx.x;
  const TileInfo ta = map_tile(P, slot, 2 * blockIdx.y, blockIdx.z);
  if (!ta.valid) return;
  const TileInfo tb = map_tile(P, slot, 2 * blockIdx.y + 1, blockIdx.z);
  // o of both heads from their support lists (one pending head recomputes both)
  if (P.from_support && P.pending[ta.tile_id] == 0 && P.pending[tb.tile_id] == 0) return;
  // Lists from the tau pass, clamped so that no workspace content sends a read outside them.
  const int cnt_a = list_count(P, ta);
  const int cnt_b = list_count(P, tb);
  const int* list_a = P.list + ta.tile_id * P.nkt_max;
  const int* list_b = P.list + tb.tile_id * P.nkt_max;
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * D * 2;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kPairKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kPairVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 8);  // one arrival per p warp of the head
    }
    mbar_init(&sm.o_full, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // warp 0 streams both query tiles and the key tiles, warp 2 the value tiles
      const bool keys = warp == 0;
      const CUtensorMap* map = keys ? &tmk : &tmv;
      const int stages = keys ? kPairKStages : kPairVStages;
      __nv_bfloat16* ring = keys ? sm.k[0] : sm.v[0];
      uint64_t* full = keys ? sm.k_full : sm.v_full;
      uint64_t* empty = keys ? sm.k_empty : sm.v_empty;
      const int krow0 = static_cast<int>(ta.khead + ta.seq_start);
      if (keys) {
        mbar_expect_tx(&sm.q_full, 2 * kTileBytes);
        const int qa = static_cast<int>(ta.qhead + ta.seq_start + ta.row0);
        const int qb = static_cast<int>(tb.qhead + tb.seq_start + tb.row0);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(sm.q[0] + h * kTile * 64, &tmq, &sm.q_full, h * 64, qa);
          tma_load_2d(sm.q[1] + h * kTile * 64, &tmq, &sm.q_full, h * 64, qb);
        }
      }
      UnionWalk walk{list_a, list_b, cnt_a, cnt_b, 0, 0, ta.nkt, P.no_mask};
      int kt;
      bool in_a, in_b;
      int issued = 0;
      for (int u = 0; walk.next(kt, in_a, in_b); ++u) {
        const int s = u % stages;
        if (u >= stages && !mbar_wait(&empty[s], ((u / stages) - 1) & 1, abort, P.status)) break;
        mbar_expect_tx(&full[s], kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d(ring + s * kTile * D + h * kTile * 64, map, &full[s], h * 64,
                      krow0 + kt * kTile);
        issued = u + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int u = (issued > stages ? issued - stages : 0); u < issued; ++u)
        mbar_wait(&full[u % stages], (u / stages) & 1, abort, P.status);
      if (keys) mbar_wait(&sm.q_full, 0, abort, P.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, D, false, true);
      // descriptors of both query tiles for every 16-wide slice of d, and the per-slice byte
      // offsets inside a key tile (K-major) and a value tile (MN-major)
      uint64_t qdesc[2][D / 16];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16)
          qdesc[x][k16] = kmajor_desc(smem_u32(sm.q[x]), kTile, k16);
      const uint64_t kdesc0 = kmajor_desc(smem_u32(sm.k[0]), kTile, 0);
      const uint64_t vdesc0 = value_desc(smem_u32(sm.v[0]), 0);
      auto issue_s = [&](int x, int ks) {  // S_X = Q_X K^T from key stage ks
        const uint64_t kd = desc_add(kdesc0, static_cast<uint32_t>(ks) * kTileBytes);
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16)
          mma_ss(tmem + static_cast<uint32_t>(x * 128), qdesc[x][k16],
                 desc_add(kd, static_cast<uint32_t>((k16 >> 2) * kTile * 128 + (k16 & 3) * 32)),
                 idesc_s, k16 > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[x]);
      };
      auto issue_pv = [&](int x, int vs, bool first) {  // O_X += P_X V from value stage vs
        const uint64_t vd = desc_add(vdesc0, static_cast<uint32_t>(vs) * kTileBytes);
        const uint32_t sx = tmem + static_cast<uint32_t>(x * 128);
#pragma unroll
        for (int k16 = 0; k16 < kTile / 16; ++k16)
          mma_ts(tmem + kPairColO + static_cast<uint32_t>(x * 128),
                 sx + static_cast<uint32_t>(64 * (k16 >> 2) + 8 * (k16 & 3)),
                 desc_add(vd, static_cast<uint32_t>(k16) * 2048u), idesc_o,
                 (first && k16 == 0) ? 0u : 1u);
      };
      bool ok = mbar_wait(&sm.q_full, 0, abort, P.status);
      UnionWalk walk{list_a, list_b, cnt_a, cnt_b, 0, 0, ta.nkt, P.no_mask};
      int kt;
      bool cur_a = false, cur_b = false;
      bool more = walk.next(kt, cur_a, cur_b);
      int done_a = 0, done_b = 0;  // PV products issued per head
      if (ok && more) {
        ok = mbar_wait(&sm.k_full[0], 0, abort, P.status);
        if (ok) {
          tc_fence_after();
          if (cur_a) issue_s(0, 0);
          if (cur_b) issue_s(1, 0);
          mma_commit(&sm.k_empty[0]);
        }
      }
      for (int u = 0; ok && more; ++u) {
        bool nx_a = false, nx_b = false;
        const bool more_nx = walk.next(kt, nx_a, nx_b);
        const int ks = (u + 1) % kPairKStages, vs = u % kPairVStages;
        // each resource is awaited just before its first use, so that whatever is ready
        // reaches the tensor pipe first
        if (!mbar_wait(&sm.v_full[vs], (u / kPairVStages) & 1, abort, P.status)) break;
        if (cur_a) {
          if (!mbar_wait(&sm.p_full[0], done_a & 1, abort, P.status)) break;
          tc_fence_after();
          issue_pv(0, vs, done_a == 0);
          ++done_a;
        }
        if (more_nx &&
            !mbar_wait(&sm.k_full[ks], ((u + 1) / kPairKStages) & 1, abort, P.status))
          break;
        tc_fence_after();
        if (nx_a) issue_s(0, ks);
        if (cur_b) {
          if (!mbar_wait(&sm.p_full[1], done_b & 1, abort, P.status)) break;
          tc_fence_after();
          issue_pv(1, vs, done_b == 0);
          ++done_b;
        }
        if (nx_b) issue_s(1, ks);
        mma_commit(&sm.v_empty[vs]);
        if (more_nx) mma_commit(&sm.k_empty[ks]);
        cur_a = nx_a;
        cur_b = nx_b;
        more = more_nx;
      }
      mma_commit(&sm.o_full);  // arrives once every MMA issued so far has completed
    }
  } else if (warp >= kScoreWarp0) {
    const int x = (warp - kScoreWarp0) >> 3;  // head A or B
    const TileInfo& t = x ? tb : ta;
    const int cnt = x ? cnt_b : cnt_a;
    const int* list = x ? list_b : list_a;
    const int quarter = warp & 3;
    const int half = ((warp - kScoreWarp0) >> 2) & 1;  // keys 64 half .. 64 half + 63
    const int r = quarter * 32 + lane;
    const bool row_ok = r < t.nrows;
    const int pos = t.row0 + r;
    const int jmax = row_ok ? (P.causal ? pos + 1 : t.seq_len) : 0;
    const float tau = row_ok ? P.tau[t.qhead + t.seq_start + pos] : INFINITY;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t sx = tmem + lane_off + static_cast<uint32_t>(x * 128);
    for (int i = 0; i < cnt; ++i) {
      const int kt = list_tile(P, list, i, t.nkt);
      if (!mbar_wait(&sm.s_full[x], i & 1, abort, P.status)) break;
      tc_fence_after();
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int c0 = half * 64 + q2 * 32;  // S column == key offset in the tile
        uint32_t u[32];
        tmem_ld32(sx + static_cast<uint32_t>(c0), u);
        uint32_t pk[16];
        p_row32<BK>(u, P.c, tau, P.beta, kt * kTile + c0, jmax, pk);
        // keys c0 .. c0 + 31 as 16 packed columns over S columns this warp has already read
        tmem_st16(sx + static_cast<uint32_t>(half * 64 + q2 * 16), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[x]);
    }
    // epilogue: this warp's half of O_X's columns, from TMEM to global memory
    const bool o_ok = mbar_wait(&sm.o_full, 0, abort, P.status);
    tc_fence_after();
    constexpr int kHalfD = D / 2;
    const int64_t oe = (t.qhead + t.seq_start + pos) * D + half * kHalfD;  // element offset
    // Full tiles at d = 128: the four warps of a (head, half) stage their 32 rows x 64 columns
    // in the key ring (idle once o_full has arrived: every key tile loaded has been used) as one
    // 128-row box in the 128-byte swizzled layout, and one TMA store writes it.  box_tile is the
    // same for the four warps (it depends on the head only), so all four reach the barrier; the
    // store is issued only if every one of them staged its rows (no timeout, no abort).
    const bool box_tile = D == 128 && cnt > 0 && t.nrows == kTile && !P.out_f32;
    if (box_tile) {
      const bool staged = o_ok && !*abort;
      const int box = (warp - kScoreWarp0) >> 2;  // (head, half) = (box >> 1, box & 1)
      unsigned char* stage = reinterpret_cast<unsigned char*>(sm.k[0]) + box * (kTile * 128);
#pragma unroll
      for (int c0 = 0; c0 < (staged ? kHalfD : 0); c0 += 32) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + kPairColO + static_cast<uint32_t>(x * 128 + half * kHalfD + c0),
                  u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // 16-byte chunk (c0 / 8 + e) of row r, swizzled
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(u[8 * e + 0]), __uint_as_float(u[8 * e + 1]));
          w.y = pack_bf16x2(__uint_as_float(u[8 * e + 2]), __uint_as_float(u[8 * e + 3]));
          w.z = pack_bf16x2(__uint_as_float(u[8 * e + 4]), __uint_as_float(u[8 * e + 5]));
          w.w = pack_bf16x2(__uint_as_float(u[8 * e + 6]), __uint_as_float(u[8 * e + 7]));
          const int chunk = (c0 / 8 + e) ^ (r & 7);
          *reinterpret_cast<uint4*>(stage + r * 128 + chunk * 16) = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      uint32_t all_staged;
      asm volatile(
          "{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n"
          " barrier.red.and.pred q, %2, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
          : "=r"(all_staged)
          : "r"(static_cast<int>(staged)), "r"(1 + box)
          : "memory");
      if (all_staged && quarter == 0 && lane == 0)
        tma_store_2d_and_wait(&tmo, stage, half * kHalfD,
                              static_cast<int>(t.qhead + t.seq_start + t.row0));
    } else if (o_ok && !*abort && cnt == 0 && row_ok) {  // no listed tile (failed tau pass only)
      zero_out(P, oe, kHalfD);
    } else if (o_ok && !*abort) {
#pragma unroll 1
      for (int c0 = 0; c0 < kHalfD; c0 += 32) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + kPairColO + static_cast<uint32_t>(x * 128 + half * kHalfD + c0),
                  u);
        if (row_ok) store_out32(P, oe + c0, u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- output from the supports --
// out_support_kernel: o_i = sum_j p_ij v_j over the support list the tau pass recorded for row i
// (record_support), for every query tile that is not pending.  One CTA of 128 threads per query
// tile; 8 lanes per row, each owning d / 8 consecutive columns (a value row is one contiguous
// 2 d-byte read by the 8 lanes), 16 rows at a time, two entries of a row loaded before either is
// accumulated.  Keys, offsets and counts are clamped to the tile's list and sequence, so an
// unfilled workspace cannot send a read outside them.
constexpr int kSupThreads = 128;

template <int D>
__global__ void __launch_bounds__(kSupThreads)
    out_support_kernel(Problem P) {
  const int slot = gridDim.x - 1 - blockIdx.x;
  const TileInfo t = map_tile(P, slot, blockIdx.y, blockIdx.z);
  if (!t.valid || P.pending[t.tile_id] != 0) return;
  constexpr int kCols8 = D / 8;      // columns per lane
  constexpr int kVec = kCols8 / 8;   // 16-byte vectors per lane and value row
  const int l8 = threadIdx.x & 7;
  const int2* list = P.sup + t.tile_id * kSupPerTile;
  const __nv_bfloat16* vb =
      static_cast<const __nv_bfloat16*>(P.v) + (t.khead + t.seq_start) * D + l8 * kCols8;
  for (int r = threadIdx.x >> 3; r < t.nrows; r += kSupThreads / 8) {
    const int64_t row = t.qhead + t.seq_start + t.row0 + r;
    const int idx = P.sup_idx[row];
    const int first = min(idx & 0xffff, kSupPerTile);
    const int n = min(idx >> 16, kSupPerTile - first);
    float acc[kCols8];
#pragma unroll
    for (int i = 0; i < kCols8; ++i) acc[i] = 0.f;
    for (int e = 0; e < n; e += 2) {
      const int2 a = list[first + e];
      const int2 b = (e + 1 < n) ? list[first + e + 1] : make_int2(a.x, 0);
      const int ja = min(max(a.x, 0), t.seq_len - 1), jb = min(max(b.x, 0), t.seq_len - 1);
      const float pa = __int_as_float(a.y), pb = __int_as_float(b.y);
      uint4 wa[kVec], wb[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        wa[u] = __ldg(reinterpret_cast<const uint4*>(vb + static_cast<int64_t>(ja) * D) + u);
        wb[u] = __ldg(reinterpret_cast<const uint4*>(vb + static_cast<int64_t>(jb) * D) + u);
      }
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const uint32_t xa[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
        const uint32_t xb[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xa[h]));
          const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xb[h]));
          acc[8 * u + 2 * h] = fmaf(pb, fb.x, fmaf(pa, fa.x, acc[8 * u + 2 * h]));
          acc[8 * u + 2 * h + 1] = fmaf(pb, fb.y, fmaf(pa, fa.y, acc[8 * u + 2 * h + 1]));
        }
      }
    }
    const int64_t oe = row * D + l8 * kCols8;  // element offset of this lane's columns
    if (P.out_f32) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(P.out) + oe);
#pragma unroll
      for (int u = 0; u < 2 * kVec; ++u)
        dst[u] = make_uint4(__float_as_uint(acc[4 * u]), __float_as_uint(acc[4 * u + 1]),
                            __float_as_uint(acc[4 * u + 2]), __float_as_uint(acc[4 * u + 3]));
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.out) + oe);
#pragma unroll
      for (int u = 0; u < kVec; ++u)
        dst[u] = make_uint4(pack_bf16x2(acc[8 * u], acc[8 * u + 1]),
                            pack_bf16x2(acc[8 * u + 2], acc[8 * u + 3]),
                            pack_bf16x2(acc[8 * u + 4], acc[8 * u + 5]),
                            pack_bf16x2(acc[8 * u + 6], acc[8 * u + 7]));
    }
  }
}

// ------------------------------------------------------------------ routing scores (tcgen05) --
// route_scores_kernel: z[b, h, i, c] = zscale * q_i . sigma_c (sigma: the chunk summaries of kv
// head floor(h / G)) for one 128-row x 128-chunk tile per CTA: the query and summary tiles come
// in by TMA, one thread issues the d / 16 tcgen05.mma of the 128 x 128 product into TMEM, and the
// four warps read their 32 rows back (thread = row) and store the row's 128 values (fp32, clipped
// to the rows and chunks of the head).  Boxes past a head's rows read the next head's rows (never
// stored) or, past the tensor, zeros.  Every wait is bounded as in the other kernels.
constexpr int kRouteThreads = 128;

template <int D>
struct RouteSmem {
  alignas(1024) __nv_bfloat16 q[kTile * D];
  alignas(1024) __nv_bfloat16 s[kTile * D];
  uint64_t full;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_scores_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tms, float* __restrict__ z, int T,
                        int nc, int Hq, int G, int Hkv, float zscale, int* status) {
  extern __shared__ unsigned char smem_raw[];
  RouteSmem<D>& sm = *reinterpret_cast<RouteSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.z, b = bh / Hq, h = bh % Hq;
  const int i0 = blockIdx.x * kTile, c0 = blockIdx.y * kTile;
  volatile int* abort = &sm.abort;
  constexpr uint32_t kTileBytes = kTile * D * 2;
  if (tid == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(&sm.tmem_base, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (tid == 0) {
    mbar_expect_tx(&sm.full, 2 * kTileBytes);
    const int qrow = bh * T + i0;
    const int srow = (b * Hkv + h / G) * nc + c0;
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_2d(sm.q + hh * kTile * 64, &tmq, &sm.full, hh * 64, qrow);
      tma_load_2d(sm.s + hh * kTile * 64, &tms, &sm.full, hh * 64, srow);
    }
    if (mbar_wait(&sm.full, 0, abort, status)) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
#pragma unroll
      for (int k16 = 0; k16 < D / 16; ++k16)
        mma_ss(tmem, kmajor_desc(smem_u32(sm.q), kTile, k16), kmajor_desc(smem_u32(sm.s), kTile, k16),
               idesc, k16 > 0 ? 1u : 0u);
      mma_commit(&sm.done);
    } else {
      mbar_wait(&sm.full, 0, abort, status);  // bounded: the copies land before the CTA exits
    }
  }
  __syncwarp();
  const bool ok = mbar_wait(&sm.done, 0, abort, status) && !*abort;
  tc_fence_after();
  const int r = warp * 32 + lane;  // row of the tile == TMEM lane
  float* zr = z + (static_cast<int64_t>(bh) * T + i0 + r) * nc + c0;
  const bool row_ok = i0 + r < T;
#pragma unroll 1
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t u[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(32 * cc), u);
    if (!ok || !row_ok) continue;
    const int cb = c0 + 32 * cc;
    if (cb + 32 <= nc && (nc & 3) == 0) {  // whole 32-chunk run, 16-byte aligned row
      float4* dst = reinterpret_cast<float4*>(zr + 32 * cc);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(zscale * __uint_as_float(u[4 * e]), zscale * __uint_as_float(u[4 * e + 1]),
                             zscale * __uint_as_float(u[4 * e + 2]),
                             zscale * __uint_as_float(u[4 * e + 3]));
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (cb + e < nc) zr[32 * cc + e] = zscale * __uint_as_float(u[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------------------ host side --

int64_t q_rows(const Problem& P) { return static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hq * P.T; }
int64_t kv_rows(const Problem& P) { return static_cast<int64_t>(P.cu ? 1 : P.B) * P.Hkv * P.T; }
int64_t warm_rows(const Problem& P) {
  return static_cast<int64_t>(P.B) * P.Hkv * P.warm_levels * kTile;
}

dim3 tile_grid(const Problem& P) { return dim3(P.slots, P.Hq, P.cu ? 1 : P.B); }

// Keys above this many bytes do not stay in L2 (126 MB) next to the streaming queries.
constexpr int64_t kKeysInL2Bytes = 96ll << 20;

template <int D, int BK>
cudaError_t launch_tau_t(const Problem& P0, cudaStream_t s) {
  Problem P = P0;
  P.kv_major = kv_rows(P) * D * 2 > kKeysInL2Bytes ? 1 : 0;
  CUtensorMap mq, mk, mw;
  cudaError_t e = make_map(&mq, P.q, q_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mk, P.k, kv_rows(P), D);
  // warm-up tiles: [groups * levels * 128, d]; without them the map is never read
  if (e == cudaSuccess)
    e = P.warm_levels > 0 ? make_map(&mw, P.warm, warm_rows(P), D)
                          : make_map(&mw, P.k, kv_rows(P), D);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(TauSmem<D, BK>) + 1024;
  auto kern = tau_tc_kernel<D, BK>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = device_sms(&sms);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = static_cast<int64_t>(P.slots) * P.Hq * (P.cu ? 1 : P.B);
  kern<<<static_cast<unsigned>(std::min<int64_t>(ntiles, sms)), tau_threads(D, BK), smem, s>>>(
      mq, mk, mw, P);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_sweep_t(const Problem& P, int num_ctas, cudaStream_t s) {
  CUtensorMap mk;
  cudaError_t e = make_map(&mk, P.k, kv_rows(P), D);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(SweepSmem<D>) + 1024;
  auto kern = tau_tc_sweep_kernel<D, BK>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<num_ctas, kTauThreads, smem, s>>>(mk, P);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_out_t(const Problem& P, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  cudaError_t e = make_map(&mq, P.q, q_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mk, P.k, kv_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mv, P.v, kv_rows(P), D);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(OutSmem<D>) + 1024;
  auto kern = out_tc_kernel<D, BK>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<tile_grid(P), kOutThreads, smem, s>>>(mq, mk, mv, P);
  return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_out_pair_t(const Problem& P, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mo;
  cudaError_t e = make_map(&mq, P.q, q_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mk, P.k, kv_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mv, P.v, kv_rows(P), D);
  if (e == cudaSuccess) e = make_map(&mo, P.out, q_rows(P), D);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(PairSmem<D>) + 1024;
  auto kern = out_pair_kernel<D, BK>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(P.slots, P.Hq / 2, P.cu ? 1 : P.B), kPairThreads, smem, s>>>(mq, mk, mv, mo, P);
  return cudaGetLastError();
}

cudaError_t launch_support_t(const Problem& P, cudaStream_t s) {
  if (P.d == 64)
    out_support_kernel<64><<<tile_grid(P), kSupThreads, 0, s>>>(P);
  else
    out_support_kernel<128><<<tile_grid(P), kSupThreads, 0, s>>>(P);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_route_scores_d(const void* q, const void* sig, float* z, int B, int Hq,
                                  int Hkv, int T, int nc, float zscale, int* status,
                                  cudaStream_t s) {
  CUtensorMap mq, ms;
  cudaError_t e = make_map(&mq, q, static_cast<int64_t>(B) * Hq * T, D);
  if (e == cudaSuccess) e = make_map(&ms, sig, static_cast<int64_t>(B) * Hkv * nc, D);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(RouteSmem<D>) + 1024;
  auto kern = route_scores_kernel<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((T + kTile - 1) / kTile, (nc + kTile - 1) / kTile, B * Hq);
  kern<<<grid, kRouteThreads, smem, s>>>(mq, ms, z, T, nc, Hq, Hq / Hkv, Hkv, zscale, status);
  return cudaGetLastError();
}

#define EA_TC_DISPATCH(FN)                                          \
  do {                                                              \
    const int bk = beta_kind(P.beta);                               \
    if (P.d == 64) {                                                \
      if (bk == kBetaOne) return FN<64, kBetaOne>(P, s);            \
      if (bk == kBetaTwo) return FN<64, kBetaTwo>(P, s);            \
      if (bk == kBetaNear3) return FN<64, kBetaNear3>(P, s);    \
      return FN<64, kBetaGeneral>(P, s);                            \
    }                                                               \
    if (bk == kBetaOne) return FN<128, kBetaOne>(P, s);             \
    if (bk == kBetaTwo) return FN<128, kBetaTwo>(P, s);             \
    if (bk == kBetaNear3) return FN<128, kBetaNear3>(P, s);     \
    return FN<128, kBetaGeneral>(P, s);                             \
  } while (0)

}  // namespace

cudaError_t launch_tau_tc(const Problem& P, cudaStream_t s) { EA_TC_DISPATCH(launch_tau_t); }

cudaError_t launch_tau_tc_fallback(const Problem& P, int num_ctas, cudaStream_t s) {
  const int bk = beta_kind(P.beta);
  if (P.d == 64) {
    if (bk == kBetaOne) return launch_sweep_t<64, kBetaOne>(P, num_ctas, s);
    if (bk == kBetaTwo) return launch_sweep_t<64, kBetaTwo>(P, num_ctas, s);
    if (bk == kBetaNear3) return launch_sweep_t<64, kBetaNear3>(P, num_ctas, s);
    return launch_sweep_t<64, kBetaGeneral>(P, num_ctas, s);
  }
  if (bk == kBetaOne) return launch_sweep_t<128, kBetaOne>(P, num_ctas, s);
  if (bk == kBetaTwo) return launch_sweep_t<128, kBetaTwo>(P, num_ctas, s);
  if (bk == kBetaNear3) return launch_sweep_t<128, kBetaNear3>(P, num_ctas, s);
  return launch_sweep_t<128, kBetaGeneral>(P, num_ctas, s);
}
cudaError_t launch_out_support(const Problem& P, cudaStream_t s) { return launch_support_t(P, s); }

cudaError_t launch_route_scores_tc(const void* q, const void* sig, float* z, int B, int Hq,
                                   int Hkv, int T, int d, int nc, float zscale, int* status,
                                   cudaStream_t s) {
  return d == 64 ? launch_route_scores_d<64>(q, sig, z, B, Hq, Hkv, T, nc, zscale, status, s)
                 : launch_route_scores_d<128>(q, sig, z, B, Hq, Hkv, T, nc, zscale, status, s);
}

cudaError_t launch_out_tc(const Problem& P, cudaStream_t s) {
  // heads 2 j and 2 j + 1 share their key/value head when the group size is even
  if (P.G % 2 == 0) EA_TC_DISPATCH(launch_out_pair_t);
  EA_TC_DISPATCH(launch_out_t);
}

}  // namespace ea
