// common.cuh -- problem description, query-tile map, and the per-row candidate buffer + tau
// solve shared by the tau-pass kernels of the entmax attention library.
//
// Notation (AdaSplash: Adaptive Sparse Flash Attention, "AdaSplash with Block Masking"):
//   raw score   r_ij = q_i . k_j                      (fp32 accumulate)
//   z_ij        = c * r_ij,  c = (alpha - 1) / sqrt(d)
//   p_ij        = [z_ij - tau_i]_+ ^ beta,  beta = 1 / (alpha - 1)
// Because p_ij <= 1, tau_i >= m_i - 1 with m_i = max_j z_ij, so only keys with z > m - 1 can
// carry p > 0.  The tau pass keeps exactly those keys ("candidates") per row while it sweeps
// the key tiles, then runs the bracketed Halley + bisection search of the "Triton Entmax
// (Optimized Entmax Activation)" section over the candidates alone.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

namespace ea {

constexpr int kTile = 128;      // query-tile rows and key-tile keys (block-mask granularity)
constexpr int kSeg = 4;         // key segments per row (keys 32 g .. 32 g + 31 of every key tile),
                                // each with its own running max and candidate buffer
constexpr int kCand = 16;       // candidate slots per (row, segment) held in shared memory: the
                                // default; kernels with shared memory to spare take more
constexpr int kCols = kSeg * kTile;  // (row, segment) columns of the candidate buffers
constexpr int kXchWarps = 16;  // warps feeding candidates per CTA (one exchange row each)
constexpr int kExchangeMax = 2;  // up to this many rows of a warp take the exchange row
constexpr int kMaxWords = 64;   // mask words per query tile the kernels support (T <= 262144)

// beta = 1 and 2 have exact closed forms; kBetaNear3 is beta within kNearIntFrac of 3 (alpha
// near 4/3, e.g. the fp32 value of 1.333: beta = 3.003); the rest is general.
enum BetaKind { kBetaOne = 0, kBetaTwo = 1, kBetaGeneral = 2, kBetaNear3 = 3 };
constexpr float kNearIntFrac = 0.004f;

// Everything a kernel needs; passed by value.
struct Problem {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* tau;
  uint32_t* mask;
  const int32_t* cu;   // nullptr = fixed length
  int B, Hq, Hkv, T, d, G;
  int causal;
  int n_iter;
  float alpha;
  float beta;          // 1 / (alpha - 1)
  float c;             // (alpha - 1) / sqrt(d)
  int slots;           // query tiles (slots) per head
  int W;               // mask words per query tile
  int nkt_max;         // stride of a compact list
  // workspace
  int* list;           // [tiles][nkt_max]
  int* count;          // [tiles]
  int* queue;          // [tiles] overflow queue
  int* queue_count;    // 1 int
  int* status;         // per-device status word
  int force_fallback;  // every tile takes the overflow path
  int test_stall;      // test hook: the tensor-core tau kernel never requests its query tile
  int no_mask;         // no block mask: the tau pass writes neither mask nor lists, and the
                       // output pass visits every causally valid key tile
  // warm-up keys of the tensor-core tau pass (workspace; see warm_level)
  float* norms;        // [kv rows] squared key norms
  void* warm;          // [groups][warm_levels][128][d] bf16: per (batch or sequence, kv head)
                       // and level, the 128 keys of largest norm of the level's key range
  int warm_levels;     // levels per group; 0 = no warm-up keys
  int kv_major;        // tau pass tile order: 1 = all query tiles of one key group before the
                       // next (keys larger than L2), 0 = slot-major (see tau_tile)
  // Output from the supports (ENTMAX_ATTN_FLAG_SUPPORT): with record_support the tensor-core
  // tau pass records each row's support -- the keys with p > 0 and their p -- from its candidate
  // buffers, or for a query tile whose buffers overflowed from an extra sweep of the overflow
  // kernel, and sets pending[tile] to 0 for a recorded tile, 1 where the tile output pass must
  // compute o (more support entries than a tile's list holds).  With from_support the output
  // pass computes o of the recorded tiles from their lists and runs the tile pass over the
  // pending ones only.
  int* pending;        // [tiles] (workspace)
  int2* sup;           // [tiles][kSupPerTile] (key of the sequence, bits of p) (workspace)
  int* sup_idx;        // [q rows]: first entry | (entries << 16) of the row in its tile's list
  int record_support;
  int from_support;
  int out_f32;         // out is fp32 (bf16 inputs, tensor-core path): no rounding of o to bf16
  // FP8 screen (entmax_attn_tau_pass_screened): per query tile the key tiles the tensor-core
  // tau kernel visits (ascending, [tiles][nkt_max]) and their count; null = every causal tile
  const int* scr_list;
  const int* scr_count;
};

// Support entries a query tile's list holds (16 per row on average; rows may use more).
constexpr int kSupPerTile = 2048;

struct TileInfo {
  int valid;        // 0 = unused slot of a packed batch
  int h;            // q head
  int qt;           // query tile index inside its sequence
  int seq_start;    // first packed token of the sequence (0 for fixed length)
  int seq_len;
  int row0;         // position (inside the sequence) of the tile's first row
  int nrows;        // rows of this tile (<= 128)
  int nkt;          // key tiles the tile visits: qt + 1 causal, all of the sequence otherwise
  int64_t qhead;    // row offset of this (batch, q head) in q / out / tau
  int64_t khead;    // row offset of this (batch, kv head) in k / v
  int64_t tile_id;  // (batch * Hq + h) * slots + slot
  int grp;          // (batch or sequence) * Hkv + kv head: the key group of the tile
};

// Maps a (slot, head, batch) grid coordinate to its query tile.  For a packed batch, sequence s
// owns slots floor(cu[s] / 128) + s + [0, ceil(len_s / 128)); the base is nondecreasing in s,
// so the sequence of a slot is found by binary search (batch must be 0 then).
__device__ __forceinline__ TileInfo map_tile(const Problem& P, int slot, int h, int b) {
  TileInfo t;
  t.h = h;
  if (P.cu == nullptr) {
    t.seq_start = 0;
    t.seq_len = P.T;
    t.qt = slot;
    t.qhead = ((int64_t)b * P.Hq + h) * P.T;
    t.khead = ((int64_t)b * P.Hkv + h / P.G) * P.T;
    t.grp = b * P.Hkv + h / P.G;
  } else {
    int lo = 0, hi = P.B - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (P.cu[mid] / kTile + mid <= slot) lo = mid;
      else hi = mid - 1;
    }
    t.seq_start = P.cu[lo];
    t.seq_len = P.cu[lo + 1] - P.cu[lo];
    t.qt = slot - (P.cu[lo] / kTile + lo);
    t.qhead = (int64_t)h * P.T;
    t.khead = (int64_t)(h / P.G) * P.T;
    t.grp = lo * P.Hkv + h / P.G;
  }
  const int nqt = (t.seq_len + kTile - 1) / kTile;
  t.valid = (t.qt >= 0 && t.qt < nqt);
  t.row0 = t.qt * kTile;
  t.nrows = t.valid ? min(kTile, t.seq_len - t.row0) : 0;
  t.nkt = P.causal ? t.qt + 1 : nqt;
  t.tile_id = ((int64_t)b * P.Hq + h) * P.slots + slot;
  return t;
}

// Query tile L of the tau pass's tile order.  Slot-major: the longest tiles (highest slot) of
// every head first, so that the tiles a persistent CTA takes in turn shrink as the pass runs
// out.  Key-group-major (P.kv_major, when the keys do not fit in L2): all query tiles of one
// (batch or sequence, kv head) -- its G heads, longest slot first -- before the next group, so
// that the CTAs running at a time sweep the keys of one or two groups, which stay in L2, instead
// of every group's; the load balance is a little worse (the tile lengths saw-tooth per group).
__device__ __forceinline__ TileInfo tau_tile(const Problem& P, int L, int per_slot) {
  if (P.kv_major) {
    const int per_group = P.slots * P.G;
    const int grp = L / per_group, r = L - grp * per_group;
    const int hk = grp % P.Hkv;
    return map_tile(P, P.slots - 1 - r / P.G, hk * P.G + r % P.G, grp / P.Hkv);
  }
  const int slot = P.slots - 1 - L / per_slot;
  const int hb = L % per_slot;
  return map_tile(P, slot, hb % P.Hq, hb / P.Hq);
}

// Warm-up keys.  A row's candidate threshold is (running max) - 1/c, and it is loose until the
// running max has met the row's largest scores; keys of large norm are the likeliest to give
// them.  So for every key group and level j the library keeps the 128 keys of largest norm among
// the group's first 1024 * 2^j keys, and the tau pass starts each query tile with one product
// against the widest level inside the keys that every row of the tile may attend to (all keys
// before the tile's first row when causal, the whole sequence otherwise).  Their scores are real
// scores of the row, so their max is a lower bound of the row max and the threshold stays exact.
constexpr int kWarmBase = 1024;  // keys in the range of level 0
__host__ __device__ inline int warm_levels_for(int64_t n) {
  int j = 0;
  while ((static_cast<int64_t>(kWarmBase) << j) <= n) ++j;
  return j;
}
// Level of a query tile's warm-up product, -1 for none.
__device__ __forceinline__ int warm_level(const Problem& P, const TileInfo& t) {
  const int prefix = P.causal ? t.row0 : t.seq_len;
  return min(warm_levels_for(prefix), P.warm_levels) - 1;
}

__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float* p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, int64_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// For beta = 3 + f with |f| <= kNearIntFrac: x^f = exp(f ln x) by its second-order Taylor
// polynomial in l = f ln x.  Every x the passes raise to beta lies in (0, 1] (tau >= m - 1), and
// wherever x^beta >= 1e-16 (x >= 4e-6) |l| <= 0.05, so the relative error |l|^3 / 6 stays below
// 2.2e-5; below that x^3 is itself under 1e-16 and the polynomial stays positive.  One
// logarithm instead of the logarithm and exponential of exp2(beta log2 x).
__device__ __forceinline__ float near_int_frac_pow(float x, float f) {
  const float l = f * 0.69314718f * __log2f(x);
  return fmaf(l, fmaf(0.5f, l, 1.f), 1.f);
}

// x^beta and the two lower powers needed by the Halley step, for x > 0.
template <int BK>
__device__ __forceinline__ void entmax_powers(float x, float beta, float& p0, float& p1,
                                              float& p2) {
  if (BK == kBetaOne) {
    p0 = x; p1 = 1.f; p2 = 0.f;
  } else if (BK == kBetaTwo) {
    p0 = x * x; p1 = x; p2 = 1.f;
  } else if (BK == kBetaNear3) {
    p2 = x * near_int_frac_pow(x, beta - 3.f);
    p1 = p2 * x;
    p0 = p1 * x;
  } else {
    p0 = exp2f(beta * __log2f(x));
    const float inv = __frcp_rn(x);
    p1 = p0 * inv;
    p2 = p1 * inv;
  }
}

// p = [x]_+^beta
template <int BK>
__device__ __forceinline__ float entmax_p(float x, float beta) {
  if (!(x > 0.f)) return 0.f;
  if (BK == kBetaOne) return x;
  if (BK == kBetaTwo) return x * x;
  if (BK == kBetaNear3) return (x * x) * (x * near_int_frac_pow(x, beta - 3.f));
  return exp2f(beta * __log2f(x));
}

// [x]_+^beta without a branch on the sign of x: the same values as entmax_p (x <= 0 gives 0:
// max(x, 0) is 0, and log2(0) = -inf sends exp2 to 0).
template <int BK>
__device__ __forceinline__ float entmax_p_clamped(float x, float beta) {
  const float y = fmaxf(x, 0.f);
  if (BK == kBetaOne) return y;
  if (BK == kBetaTwo) return y * y;
  if (BK == kBetaNear3) return (y * y) * (y * near_int_frac_pow(fmaxf(y, 1e-30f), beta - 3.f));
  return exp2f(beta * __log2f(y));
}

// State of the bracketed Halley + bisection search for one row: the iterate, the bracket, and
// the lengths of the last two steps.
struct Search {
  float tau, lo, hi, dx, dxold, m;

  // p_max <= 1 gives tau >= m - 1; n keys all at most m give tau <= m - n^(1 - alpha), with
  // equality when all n tie at m.  The upper end is raised by a rounding margin: a step that
  // lands on a root at that end (exactly so for alpha = 2, where f is linear in tau) carries the
  // rounding of tau - f / f', a few ulps of |m| + 1, and without the margin it would fall just
  // outside the bracket at every step and leave tau to bisection.
  __device__ __forceinline__ void init(float m_, int n, float alpha) {
    m = m_;
    lo = m - 1.f;
    hi = m - exp2f((1.f - alpha) * __log2f((float)n)) + 8.f * FLT_EPSILON * (fabsf(m) + 1.f);
    tau = lo;
    dx = dxold = hi - lo;
  }

  // True once the last step moved tau by no more than rounding, measured against the larger of
  // |tau| (what fp32 can resolve) and m - tau (the size of the differences z - tau that p is
  // made of, small for long near-uniform rows when alpha > 2): later steps can then only move
  // it by a few ulps.
  __device__ __forceinline__ bool settled() const {
    return dx <= 4.f * FLT_EPSILON * fmaxf(fabsf(tau), m - tau);
  }

  // One step, given the sums over the keys with z > tau of (z - tau)^beta, ^(beta-1) and
  // ^(beta-2): f = S0 - 1, f' = -beta S1, f'' = beta (beta - 1) S2.  The bracket is narrowed by
  // the sign of f.  The proposal is the Halley step when its denominator 2 f'^2 - f f'' is
  // positive and finite (it then points at the root), else the Newton step.  It is taken if it
  // lies in the closed bracket and is either within rounding of tau or at most half as long as
  // the step before last (the progress test of the safeguarded Newton method "rtsafe",
  // Numerical Recipes); otherwise the bracket midpoint is taken.
  template <int BK>
  __device__ __forceinline__ void step(float s0, float s1, float s2, float beta) {
    const float f = s0 - 1.f;
    const float f1 = -beta * s1;
    const float f2 = (BK == kBetaOne) ? 0.f : beta * (beta - 1.f) * s2;
    if (f > 0.f) lo = tau;
    else hi = tau;
    const float den = 2.f * f1 * f1 - f * f2;
    // the quotient is only a proposal (the bracket test below guards it): fast division
    float nt = (den > 0.f && den < INFINITY) ? tau - __fdividef(2.f * f * f1, den)
                                             : tau - __fdividef(f, f1);
    const float len = fabsf(nt - tau);
    const bool small = len <= 4.f * FLT_EPSILON * fmaxf(1.f, fabsf(tau));
    if (!(nt >= lo && nt <= hi && (small || len <= 0.5f * dxold))) nt = 0.5f * (lo + hi);
    dxold = dx;
    dx = fabsf(nt - tau);
    tau = nt;
  }
};

// ---------------------------------------------------------------------------------------------
// Candidate buffers: for every (row r, segment g) -- column c = g * 128 + r -- up to NC
// (raw score, key id) pairs in shared memory, entry e at [e * kCols + c], so that the 32 rows
// of a warp hit 32 distinct banks whatever their fill levels.  A segment owns the keys 32 g ..
// 32 g + 31 of every key tile; the key id of key 128 kt + 32 g + i is 32 kt + i (kt < 2048, so it
// fits 16 bits), from which both the key tile (mask bits) and the key itself (the output gather)
// are recovered.
// ---------------------------------------------------------------------------------------------
template <int NC>
struct alignas(16) CandSmemT {
  static_assert(NC % 4 == 0, "the solve splits a buffer over 4 lanes");
  static_assert(NC <= 32, "at most one candidate slot per lane in the cooperative insertion");
  static constexpr int kSlots = NC;
  float xrow[kXchWarps][32];  // per-warp exchange rows of feed_warp (first: 16-byte aligned)
  float s[NC * kCols];
  uint16_t kt[NC * kCols];
  float rowmax[kTile];  // running max of the row over all segments (raw); see feed_warp
  float tau_r[kTile];   // the row's tau once solved (read by record_support)
  int sup_n[kTile];     // support entries of each row, then their first position in the list
  int sup_over;         // the tile's supports do not fit its list
  float m[kCols];       // segment max of raw scores
  float floor_[kCols];  // pruning floor (raw); -inf when the segment was never pruned
  int cnt[kCols];
  int lost[kCols];
  uint32_t words[kMaxWords];
  int wbase[kMaxWords];  // list position of each mask word's first active key tile
  int fallback;         // some row of the tile needs the overflow path
};
using CandSmem = CandSmemT<kCand>;

// max of three floats in one instruction
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max of x[o .. o + 16)
template <int N>
__device__ __forceinline__ float max16(const float (&x)[N], int o) {
  const float a = max3f(x[o], x[o + 1], x[o + 2]);
  const float b = max3f(x[o + 3], x[o + 4], x[o + 5]);
  const float c = max3f(x[o + 6], x[o + 7], x[o + 8]);
  const float d = max3f(x[o + 9], x[o + 10], x[o + 11]);
  const float e = max3f(x[o + 12], x[o + 13], x[o + 14]);
  return max3f(max3f(a, b, c), max3f(d, e, x[o + 15]), -INFINITY);
}

// Shared-memory stores under a predicate, issued without a branch (the insertion loops below
// would otherwise compile to one divergent branch per key).
__device__ __forceinline__ void st_shared_if(bool p, float* addr, float v) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.shared.f32 [%1], %2;\n}" ::"r"(
          static_cast<int>(p)),
      "r"(static_cast<uint32_t>(__cvta_generic_to_shared(addr))), "f"(v)
      : "memory");
}
__device__ __forceinline__ void st_shared_if(bool p, uint16_t* addr, uint16_t v) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %0, 0;\n @q st.shared.u16 [%1], %2;\n}" ::"r"(
          static_cast<int>(p)),
      "r"(static_cast<uint32_t>(__cvta_generic_to_shared(addr))), "h"(v)
      : "memory");
}

// Candidate state of one (row, segment), held in registers by the thread that owns it.
struct RowCand {
  float m;       // running max of this segment's raw scores
  float mx;      // largest max known for the row: max(m, what other segments published)
  float thr;     // keep threshold: max(mx - 1/c, floor)
  float floor_;  // pruning floor, -inf if never raised
  float inv_c;   // 1 / c
  int cnt;
  int lost;

  __device__ __forceinline__ void init(float inv_c_) {
    m = -INFINITY;
    mx = -INFINITY;
    thr = -INFINITY;
    floor_ = -INFINITY;
    inv_c = inv_c_;
    cnt = 0;
    lost = 0;
  }

  template <class CS>
  __device__ __forceinline__ void publish(CS& cs, int col) const {
    cs.m[col] = m;
    cs.floor_[col] = floor_;
    cs.cnt[col] = cnt;
    cs.lost[col] = lost;
  }
};


// Insertion of the passing values of one lane (src, buffer column col_src) when they do not fit
// into its buffer.  Lane e < c0 holds old entry e, lane j holds value j of src's chunk (v), whose
// key id is kid0 + j.
// Old entries and new values at or below the threshold th are dropped; if more than the buffer's
// slots survive, the floor is raised by bisection to just above the (slots/2 + 1)-th largest
// value, so that the slots/2 largest survive and the buffer has room again (entries below the floor
// can only matter if tau ends up at or below it, which the solve checks).  Survivors -- old ones
// first, then new ones in key order -- are written to the front of the buffer.  Warp-uniform
// arguments; call with the whole warp converged.
template <class CS>
__device__ __forceinline__ void coop_insert(CS& cs, RowCand& rc, int src, int col_src,
                                            float v, float th, int c0, int kid0, int lane) {
  const unsigned full = 0xffffffffu;
  float fl = __shfl_sync(full, rc.floor_, src);
  const float mm = __shfl_sync(full, rc.mx, src);
  const bool have = lane < c0;
  const float vo = have ? cs.s[lane * kCols + col_src] : -INFINITY;
  const uint16_t ko = have ? cs.kt[lane * kCols + col_src] : static_cast<uint16_t>(0);
  unsigned bo = __ballot_sync(full, vo > th);
  unsigned bn = __ballot_sync(full, v > th);
  if (__popc(bo) + __popc(bn) > CS::kSlots) {
    // Bisection on [th, mm] keeps "more than kKeep above lo, at most kKeep above hi".
    constexpr int kKeep = CS::kSlots / 2;
    float lo = th, hi = mm;
    for (int it = 0; it < 24; ++it) {
      const float mid = 0.5f * (lo + hi);
      if (!(mid > lo && mid < hi)) break;  // the interval cannot shrink further in fp32
      const int n = __popc(__ballot_sync(full, vo > mid)) + __popc(__ballot_sync(full, v > mid));
      if (n > kKeep) {
        lo = mid;
      } else {
        hi = mid;
        if (n == kKeep) break;  // exactly kKeep survive: as high as the floor needs to go
      }
    }
    fl = hi;
    th = hi;
    bo = __ballot_sync(full, vo > th);
    bn = __ballot_sync(full, v > th);
  }
  const unsigned below = (1u << lane) - 1u;
  const int no = __popc(bo), nn = __popc(bn);
  __syncwarp();  // every old entry is in registers before the buffer is rewritten
  if ((bo >> lane) & 1u) {
    const int at = __popc(bo & below);
    cs.s[at * kCols + col_src] = vo;
    cs.kt[at * kCols + col_src] = ko;
  }
  if ((bn >> lane) & 1u) {
    const int at = no + __popc(bn & below);
    if (at < CS::kSlots) {
      cs.s[at * kCols + col_src] = v;
      cs.kt[at * kCols + col_src] = static_cast<uint16_t>(kid0 + lane);
    }
  }
  if (lane == src) {
    const int total = no + nn;
    rc.cnt = min(total, CS::kSlots);
    if (total > CS::kSlots) rc.lost = 1;  // only when ties at the floor could not be separated
    rc.thr = th;
    rc.floor_ = fl;
  }
}

// Feeds 32 raw scores of key tile kt (keys outside the row's range already -inf) for the 32
// (row, segment) columns of a warp; every lane of the warp must call it together.  The hot path
// is the max of each 16-key block.  A row whose chunk max passes its threshold counts its values
// above it; when that is one (the common case once the row max has settled) the value is the
// chunk max and the row's lane stores it, in parallel with every other such lane.  Rows with
// several values are, when few rows of the warp have them, handled by the whole warp: its lane
// writes the chunk to the warp's exchange row xrow (32 floats, 16-byte aligned, private to the
// warp), every lane compares one value, and a ballot gives each passing value its slot.  When
// many do (more than kExchangeMax), each lane stores its own values and only rows without room
// take the exchange path.  The threshold uses the largest max any segment of
// the row has published in cs.rowmax[row]: a lower bound of the row's max, so every key with
// z > (row max) - 1 is still kept, while records of one segment's max no longer trigger
// insertions in the others.  A stale or overwritten rowmax value only loosens the threshold.
template <int N, class CS>
__device__ __forceinline__ void feed_warp(RowCand& rc, CS& cs, float* xrow, int col,
                                          int row, int lane, const float (&x)[N], int kt) {
  static_assert(N == 32, "one value per lane in the exchange row");
  const unsigned full = 0xffffffffu;
  const float cmax = fmaxf(max16(x, 0), max16(x, 16));
  const float shared_max = *reinterpret_cast<volatile float*>(&cs.rowmax[row]);
  if (shared_max > rc.mx) {
    rc.mx = shared_max;
    rc.thr = fmaxf(rc.mx - rc.inv_c, rc.floor_);
  }
  const bool pass = cmax > rc.thr;
  const unsigned passing = __ballot_sync(full, pass);
  if (!passing) return;
  if (pass) {
    rc.m = fmaxf(rc.m, cmax);
    if (cmax > rc.mx) {
      rc.mx = cmax;
      rc.thr = fmaxf(rc.mx - rc.inv_c, rc.floor_);
      cs.rowmax[row] = cmax;  // publish to the row's other segments
    }
  }
  // Most passing chunks hold a single value above the threshold, which is then the chunk max:
  // each such lane stores it itself, all at once.  The others go on below.
  const int kid0 = kt * 32;  // key id of x[0] (see the candidate buffers)
  bool single = false;
  int incoming = 0;  // this lane's values above its threshold
  if (pass) {
    int at1 = 0;     // position of the (last) value above it
#pragma unroll
    for (int i = 0; i < N; ++i) {  // >= 1: cmax > rc.thr
      const bool up = x[i] > rc.thr;
      incoming += up ? 1 : 0;
      at1 = up ? i : at1;
    }
    if (incoming == 1 && rc.cnt < CS::kSlots) {
      cs.s[rc.cnt * kCols + col] = cmax;
      cs.kt[rc.cnt * kCols + col] = static_cast<uint16_t>(kid0 + at1);
      ++rc.cnt;
      single = true;
    }
  }
  unsigned serial = __ballot_sync(full, pass && !single);
  if (!serial) return;
  __syncwarp();  // the single-value stores are visible to the warp's lanes
  if (__popc(serial) > kExchangeMax) {
    // Many rows with several values pass (the first key tiles of a row, before its max
    // settles): each lane stores its own passing values, all lanes at once; rows without room
    // go on below.
    const bool fits = pass && !single && rc.cnt + incoming <= CS::kSlots;
    if (fits) {
      int c = rc.cnt;
#pragma unroll
      for (int i = 0; i < N; ++i) {  // fixed trip count, predicated stores: no branches
        const bool take = x[i] > rc.thr;
        st_shared_if(take, &cs.s[c * kCols + col], x[i]);
        st_shared_if(take, &cs.kt[c * kCols + col], static_cast<uint16_t>(kid0 + i));
        c += take ? 1 : 0;
      }
      rc.cnt = c;
    }
    serial = __ballot_sync(full, pass && !single && !fits);
    __syncwarp();  // these stores are visible to the lanes that read the buffers below
  }
  const unsigned below = (1u << lane) - 1u;
  for (unsigned rest = serial; rest; rest &= rest - 1u) {
    const int src = __ffs(rest) - 1;
    if (lane == src) {
      float4* d = reinterpret_cast<float4*>(xrow);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        d[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
    }
    __syncwarp();
    const float v = xrow[lane];
    const float th = __shfl_sync(full, rc.thr, src);
    const int c0 = __shfl_sync(full, rc.cnt, src);
    const int col_src = col - lane + src;
    const unsigned take = __ballot_sync(full, v > th);
    const int n = __popc(take);
    if (c0 + n <= CS::kSlots) {
      if ((take >> lane) & 1u) {
        const int at = c0 + __popc(take & below);
        cs.s[at * kCols + col_src] = v;
        cs.kt[at * kCols + col_src] = static_cast<uint16_t>(kid0 + lane);
      }
      if (lane == src) rc.cnt = c0 + n;
    } else {
      coop_insert(cs, rc, src, col_src, v, th, c0, kid0, lane);
    }
    __syncwarp();  // the exchange row is read by every lane before the next row overwrites it
  }
}

// Takes 32 scores of the warm-up keys (-inf for an unused row) into the row's threshold: the
// chunk max, lowered by 1e-5 relative (and 1e-6 absolute) so that it stays below the same
// scores as the key tiles give them whatever the rounding, raises the row max shared with the
// other segments and the threshold.  The segment max (rc.m) is left to the key tiles themselves.
template <int N, class CS>
__device__ __forceinline__ void observe_bound(RowCand& rc, CS& cs, int row,
                                              const float (&x)[N]) {
  static_assert(N == 32, "32-key chunks");
  float b = fmaxf(max16(x, 0), max16(x, 16));
  b = b - fabsf(b) * 1e-5f - 1e-6f;
  const float shared_max = *reinterpret_cast<volatile float*>(&cs.rowmax[row]);
  const float mx = fmaxf(shared_max, b);
  if (mx > rc.mx) {
    rc.mx = mx;
    rc.thr = fmaxf(rc.mx - rc.inv_c, rc.floor_);
  }
  if (b > shared_max) cs.rowmax[row] = b;
}

// Solves tau for every row of the tile from the published candidate buffers of both segments,
// writes tau and sets the tile's mask words in shared memory.  Rows are handled by groups of 4
// lanes that split a row's candidates and combine their partial sums with warp shuffles.
// nthreads must be a multiple of 32; call from all threads of the block after a
// __syncthreads() that follows publish().
template <int BK, class CS>
__device__ void solve_rows(const Problem& P, const TileInfo& t, CS& cs, int tid,
                           int nthreads) {
  const int lane4 = tid & 3;
  const int groups = nthreads >> 2;
  // Every lane runs the same number of row iterations and search steps (the shuffles need the
  // whole warp); rows past the end of the tile run on an empty candidate list and store nothing.
  for (int r = tid >> 2; r < kTile; r += groups) {
    const bool valid = r < t.nrows;
    int cnt[kSeg];
    float mraw = -INFINITY;
#pragma unroll
    for (int g = 0; g < kSeg; ++g) {
      cnt[g] = valid ? cs.cnt[g * kTile + r] : 0;
      mraw = fmaxf(mraw, cs.m[g * kTile + r]);
    }
    const float mz = valid ? P.c * mraw : 0.f;
    const int pos = t.row0 + r;
    const int n = valid ? (P.causal ? pos + 1 : t.seq_len) : 1;
    // this lane's share of the row's candidates (raw scores; -inf in empty slots), held in
    // registers for all search steps
    float raw[kSeg][CS::kSlots / 4];
#pragma unroll
    for (int g = 0; g < kSeg; ++g) {
#pragma unroll
      for (int i = 0; i < CS::kSlots / 4; ++i) {
        const int e = lane4 + 4 * i;
        raw[g][i] = (e < cnt[g]) ? cs.s[e * kCols + g * kTile + r] : -INFINITY;
      }
    }
    Search sr;
    sr.init(mz, n, P.alpha);
    for (int it = 0; it < P.n_iter; ++it) {
      const float tau = sr.tau;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
      for (int g = 0; g < kSeg; ++g) {
#pragma unroll
        for (int i = 0; i < CS::kSlots / 4; ++i) {
          const float x = P.c * raw[g][i] - tau;
          if (x > 0.f) {
            float a, b, c2;
            entmax_powers<BK>(x, P.beta, a, b, c2);
            s0 += a;
            s1 += b;
            s2 += c2;
          }
        }
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      }
      sr.step<BK>(s0, s1, s2, P.beta);
      if (__all_sync(0xffffffffu, sr.settled())) break;  // every row of the warp has converged
    }
    const float tau = sr.tau;
    if (!valid) continue;
    if (lane4 == 0) {
      P.tau[t.qhead + t.seq_start + pos] = tau;
      cs.tau_r[r] = tau;
    }
    bool bad = false;
#pragma unroll
    for (int g = 0; g < kSeg; ++g) {
      const float fl = cs.floor_[g * kTile + r];
      if (cs.lost[g * kTile + r] || (fl > -INFINITY && !(tau > P.c * fl))) bad = true;
    }
    if (bad) cs.fallback = 1;
#pragma unroll
    for (int g = 0; g < kSeg; ++g) {
#pragma unroll
      for (int i = 0; i < CS::kSlots / 4; ++i) {
        if (P.c * raw[g][i] > tau) {
          const int kt = cs.kt[(lane4 + 4 * i) * kCols + g * kTile + r] >> 5;  // key id -> tile
          atomicOr(&cs.words[kt >> 5], 1u << (kt & 31));
        }
      }
    }
  }
}

// Writes the tile's mask words and its compact list of active key tiles (ascending) and count,
// or queues the tile for the overflow path.  Call from warp 0 after a __syncthreads().
__device__ __forceinline__ void emit_tile(const Problem& P, const TileInfo& t,
                                          const uint32_t* words, int fallback, int lane) {
  if (fallback) {
    if (lane == 0) {
      const int i = atomicAdd(P.queue_count, 1);
      P.queue[i] = (int)t.tile_id;
    }
    return;
  }
  if (P.no_mask) return;
  uint32_t* mw = P.mask + t.tile_id * P.W;
  int* list = P.list + t.tile_id * P.nkt_max;
  int base = 0;
  for (int w0 = 0; w0 < P.W; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t bits = (w < P.W) ? words[w] : 0u;
    if (w < P.W) mw[w] = bits;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int at = base + incl - c;
    uint32_t b = bits;
    while (b) {
      const int bit = __ffs(b) - 1;
      b &= b - 1;
      list[at++] = w * 32 + bit;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) P.count[t.tile_id] = base;
}

// emit_tile split over many threads, in two phases with a barrier of those threads between:
// phase 1 (one warp): the overflow queue or the list position of every mask word and the count;
// phase 2 (all nthreads threads): the mask words and one list entry per set bit.
template <class CS>
__device__ __forceinline__ void emit_tile_prefix(const Problem& P, const TileInfo& t, CS& cs,
                                                 int lane) {
  if (cs.fallback) {
    if (lane == 0) {
      const int i = atomicAdd(P.queue_count, 1);
      P.queue[i] = (int)t.tile_id;
    }
    return;
  }
  if (P.no_mask) return;
  int base = 0;
  for (int w0 = 0; w0 < P.W; w0 += 32) {
    const int w = w0 + lane;
    const int c = (w < P.W) ? __popc(cs.words[w]) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (w < P.W) cs.wbase[w] = base + incl - c;
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) P.count[t.tile_id] = base;
}
template <class CS>
__device__ __forceinline__ void emit_tile_entries(const Problem& P, const TileInfo& t,
                                                  const CS& cs, int tid, int nthreads) {
  if (cs.fallback || P.no_mask) return;
  uint32_t* mw = P.mask + t.tile_id * P.W;
  int* list = P.list + t.tile_id * P.nkt_max;
  for (int w = tid; w < P.W; w += nthreads) mw[w] = cs.words[w];
  for (int i = tid; i < P.W * 32; i += nthreads) {
    const uint32_t bits = cs.words[i >> 5];
    const uint32_t bit = 1u << (i & 31);
    if (bits & bit) list[cs.wbase[i >> 5] + __popc(bits & (bit - 1u))] = i;
  }
}

// A compact-list entry forced into [0, nkt): out-of-range values (an unfilled workspace) read
// key tile 0 instead of memory outside the problem.
__device__ __forceinline__ int clamp_kt(int kt, int nkt) {
  return (kt >= 0 && kt < nkt) ? kt : 0;
}

// Number of key tiles the output pass visits for a query tile: its compact list's count, clamped
// to the tile's key range, or every causally valid key tile without the block mask.
__device__ __forceinline__ int list_count(const Problem& P, const TileInfo& t) {
  return P.no_mask ? t.nkt : min(max(P.count[t.tile_id], 0), t.nkt);
}

// Key tile of entry i of that sequence (list points at the query tile's compact list).
__device__ __forceinline__ int list_tile(const Problem& P, const int* list, int i, int nkt) {
  return P.no_mask ? i : clamp_kt(list[i], nkt);
}

// Unused slot of a packed batch: zero mask words, empty list.
__device__ __forceinline__ void emit_empty(const Problem& P, const TileInfo& t, int tid,
                                           int nthreads) {
  if (P.no_mask) return;
  for (int w = tid; w < P.W; w += nthreads) P.mask[t.tile_id * P.W + w] = 0u;
  if (tid == 0) P.count[t.tile_id] = 0;
}

}  // namespace ea
