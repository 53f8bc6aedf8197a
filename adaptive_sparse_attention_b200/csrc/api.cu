// api.cu -- the C ABI of include/entmax_attn.h: argument checks, workspace layout and caching,
// and the launch sequence of the two passes.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "entmax_attn.h"
#include "kernels.h"

// Per-device status word: kernels set ENTMAX_ATTN_ETIMEOUT here when a bounded wait gives up.
__device__ int g_entmax_status;

namespace {

thread_local char g_cuda_err[256] = "";

int cuda_fail(cudaError_t e) {
  std::snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return ENTMAX_ATTN_ECUDA;
}

}  // namespace

namespace ea {
int record_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace ea

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  int slots;      // query tiles (slots) per head
  int W;          // mask words per query tile
  int nkt_max;    // longest compact list
  int64_t tiles;  // query tiles over all (batch, head)
  int warm_levels;       // warm-up key levels per key group
  int64_t norm_rows;     // key rows with a norm slot (Hq bounds Hkv)
  int64_t q_rows;        // query rows (one support index each)
  int64_t warm_bytes;    // warm-up tiles of every key group at d = 128
};

bool make_layout(int B, int Hq, int T, int has_cu, Layout* L) {
  if (B < 1 || Hq < 1 || T < 1) return false;
  const int64_t nt = (static_cast<int64_t>(T) + ea::kTile - 1) / ea::kTile;
  const int64_t slots = has_cu ? static_cast<int64_t>(T) / ea::kTile + B : nt;
  if (slots > (1 << 24)) return false;
  L->slots = static_cast<int>(slots);
  L->W = static_cast<int>((nt + 31) / 32);
  L->nkt_max = static_cast<int>(nt);
  L->tiles = (has_cu ? 1 : static_cast<int64_t>(B)) * Hq * slots;
  L->warm_levels = ea::warm_levels_for(T);
  L->norm_rows = (has_cu ? 1 : static_cast<int64_t>(B)) * Hq * T;
  L->q_rows = L->norm_rows;
  L->warm_bytes = static_cast<int64_t>(B) * Hq * L->warm_levels * ea::kTile * 128 * 2;
  return L->tiles < (int64_t(1) << 31);
}

// Workspace: [queue_count | count[tiles] | queue[tiles] | pending[tiles] | list[tiles][nkt_max] |
// key norms | warm-up tiles | support index[q rows] | support lists[tiles][kSupPerTile]], each
// section 256-byte aligned.  The sections past the lists are optional: without the warm-up
// sections the tau pass runs without warm-up keys, without the support sections every query
// tile takes the tile output pass.
struct WsView {
  int* queue_count;
  int* count;
  int* queue;
  int* pending;
  int* list;
  float* norms;
  void* warm;
  int* sup_idx;
  int2* sup;
  size_t min_bytes;   // without the warm-up and support sections
  size_t warm_bytes;  // with the warm-up sections, without the support sections
  size_t bytes;
};

WsView ws_view(void* base, const Layout& L) {
  WsView v;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  v.queue_count = reinterpret_cast<int*>(p + off);
  off += 256;
  v.count = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * L.tiles);
  v.queue = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * L.tiles);
  v.pending = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * L.tiles);
  v.list = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * static_cast<size_t>(L.tiles) * L.nkt_max);
  v.min_bytes = off;  // everything past here is the tau pass's warm-up keys
  v.norms = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * static_cast<size_t>(L.norm_rows));
  v.warm = p + off;
  off += align256(static_cast<size_t>(L.warm_bytes));
  v.warm_bytes = off;
  v.sup_idx = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * static_cast<size_t>(L.q_rows));
  v.sup = reinterpret_cast<int2*>(p + off);
  off += align256(sizeof(int2) * static_cast<size_t>(L.tiles) * ea::kSupPerTile);
  v.bytes = off;
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_mu;

int* status_ptr(int* err) {
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    *err = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e);
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_entmax_status);
    if (e != cudaSuccess) {
      *err = cuda_fail(e);
      return nullptr;
    }
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

int num_sms() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
      v = 148;
    n[dev] = v;
  }
  return n[dev];
}

// Shared checks of both passes; fills the problem description (without workspace pointers).
int check_and_describe(const void* q, const void* k, int B, int Hq, int Hkv, int T, int d,
                       float alpha, int n_iter, int causal, const int32_t* cu, int dtype,
                       Layout* L, ea::Problem* P) {
  if (!q || !k) return ENTMAX_ATTN_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv != 0) return ENTMAX_ATTN_EINVAL;
  if (d != 64 && d != 128) return ENTMAX_ATTN_EINVAL;
  if (!std::isfinite(alpha) || !(alpha > 1.f)) return ENTMAX_ATTN_EINVAL;
  if (n_iter < 1 || n_iter > 1000) return ENTMAX_ATTN_EINVAL;
  if (dtype != ENTMAX_ATTN_FP32 && dtype != ENTMAX_ATTN_BF16) return ENTMAX_ATTN_EINVAL;
  if (causal != 0 && causal != 1) return ENTMAX_ATTN_EINVAL;
  if (!make_layout(B, Hq, T, cu != nullptr, L)) return ENTMAX_ATTN_EINVAL;
  if (L->W > ea::kMaxWords) return ENTMAX_ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || (cu && !aligned16(cu))) return ENTMAX_ATTN_EALIGN;
  const double a = static_cast<double>(alpha);
  const float beta = static_cast<float>(1.0 / (a - 1.0));
  if (!std::isfinite(beta)) return ENTMAX_ATTN_EINVAL;
  std::memset(P, 0, sizeof(*P));
  P->q = q;
  P->k = k;
  P->cu = cu;
  P->B = B;
  P->Hq = Hq;
  P->Hkv = Hkv;
  P->T = T;
  P->d = d;
  P->G = Hq / Hkv;
  P->causal = causal;
  P->n_iter = n_iter;
  P->alpha = alpha;
  P->beta = beta;
  P->c = static_cast<float>((a - 1.0) / std::sqrt(static_cast<double>(d)));
  P->slots = L->slots;
  P->W = L->W;
  P->nkt_max = L->nkt_max;
  return ENTMAX_ATTN_OK;
}

void attach_workspace(ea::Problem* P, const WsView& v) {
  P->list = v.list;
  P->count = v.count;
  P->queue = v.queue;
  P->queue_count = v.queue_count;
  P->pending = v.pending;
  P->sup_idx = v.sup_idx;
  P->sup = v.sup;
  P->norms = v.norms;
  P->warm = v.warm;
}

bool use_tensor_cores(int dtype, unsigned flags) {
  return dtype == ENTMAX_ATTN_BF16 && !(flags & ENTMAX_ATTN_FLAG_CUDA_CORES);
}

struct CachedWs {
  void* ptr = nullptr;
  size_t bytes = 0;
};
// The cached workspaces, one per (device, stream), and the lock that guards them.  A call holds
// it from the lookup until both passes are enqueued, so another host thread's call on the same
// (device, stream) cannot free (and regrow) the buffer in between.
std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, CachedWs> g_ws;

}  // namespace

extern "C" {

size_t entmax_attn_mask_words(int B, int Hq, int T, int has_cu_seqlens) {
  Layout L;
  if (!make_layout(B, Hq, T, has_cu_seqlens != 0, &L)) return 0;
  return static_cast<size_t>(L.tiles) * L.W;
}

int entmax_attn_mask_layout(int B, int Hq, int T, int has_cu_seqlens, int* tiles_per_head,
                            int* words_per_tile) {
  Layout L;
  if (!make_layout(B, Hq, T, has_cu_seqlens != 0, &L)) return ENTMAX_ATTN_EINVAL;
  if (tiles_per_head) *tiles_per_head = L.slots;
  if (words_per_tile) *words_per_tile = L.W;
  return ENTMAX_ATTN_OK;
}

size_t entmax_attn_workspace_bytes(int B, int Hq, int T, int has_cu_seqlens) {
  Layout L;
  if (!make_layout(B, Hq, T, has_cu_seqlens != 0, &L)) return 0;
  return ws_view(nullptr, L).bytes;
}

size_t entmax_attn_workspace_min_bytes(int B, int Hq, int T, int has_cu_seqlens) {
  Layout L;
  if (!make_layout(B, Hq, T, has_cu_seqlens != 0, &L)) return 0;
  return ws_view(nullptr, L).min_bytes;
}

}  // extern "C"

namespace {

// The tau pass (ENTMAX_ATTN_FLAG_SUPPORT: also the support lists and pending flags).
int tau_pass_impl(const void* q, const void* k, float* tau, uint32_t* block_mask,
                  void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int T, int d,
                  float alpha, int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                  unsigned flags, cudaStream_t stream, const int* scr_list = nullptr,
                  const int* scr_count = nullptr) {
  Layout L;
  ea::Problem P;
  int rc = check_and_describe(q, k, B, Hq, Hkv, T, d, alpha, n_iter, causal, cu_seqlens, dtype,
                              &L, &P);
  if (rc != ENTMAX_ATTN_OK) return rc;
  const bool no_mask = (flags & ENTMAX_ATTN_FLAG_NO_BLOCK_MASK) != 0;
  if (!tau || (!block_mask && !no_mask) || !workspace) return ENTMAX_ATTN_EINVAL;
  if (!aligned16(tau) || (block_mask && !aligned16(block_mask)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ENTMAX_ATTN_EALIGN;
  const WsView wv = ws_view(workspace, L);
  if (workspace_bytes < wv.min_bytes) return ENTMAX_ATTN_ENOMEM;
  int err = ENTMAX_ATTN_OK;
  P.status = status_ptr(&err);
  if (!P.status) return err;
  P.tau = tau;
  P.mask = block_mask;
  attach_workspace(&P, wv);
  P.force_fallback = (flags & ENTMAX_ATTN_FLAG_ALL_FALLBACK) ? 1 : 0;
  P.test_stall = (flags & ENTMAX_ATTN_FLAG_TEST_STALL) ? 1 : 0;
  P.no_mask = no_mask ? 1 : 0;
  P.scr_list = scr_list;
  P.scr_count = scr_count;

  cudaError_t e = cudaMemsetAsync(wv.queue_count, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((flags & ENTMAX_ATTN_FLAG_OUT_FP32) && !use_tensor_cores(dtype, flags))
    return ENTMAX_ATTN_EINVAL;  // fp32 outputs of bf16 inputs: the tensor-core path only
  P.out_f32 = (flags & ENTMAX_ATTN_FLAG_OUT_FP32) ? 1 : 0;
  if (flags & ENTMAX_ATTN_FLAG_SUPPORT) {
    if (use_tensor_cores(dtype, flags) && workspace_bytes >= wv.bytes) {
      // the tensor-core tau kernel records the supports and the pending flag of every tile
      P.record_support = 1;
    } else {
      // no support lists (CUDA-core tau kernel, or no room for them): every query tile is left
      // to the tile output pass (a nonzero flag; unused slots are skipped by it anyway)
      e = cudaMemsetAsync(wv.pending, 0xff, sizeof(int) * static_cast<size_t>(L.tiles), stream);
      if (e != cudaSuccess) return cuda_fail(e);
    }
  }
  if (use_tensor_cores(dtype, flags) && workspace_bytes >= wv.warm_bytes) {
    P.warm_levels = L.warm_levels;
    e = ea::launch_warm(P, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  e = use_tensor_cores(dtype, flags) ? ea::launch_tau_tc(P, stream)
                                     : ea::launch_tau_simt(P, dtype, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  if (use_tensor_cores(dtype, flags)) {
    const int64_t ctas = std::min<int64_t>(L.tiles, num_sms());
    e = ea::launch_tau_tc_fallback(P, static_cast<int>(ctas), stream);
  } else {
    const int64_t ctas = std::min<int64_t>(L.tiles, 2 * num_sms());
    e = ea::launch_tau_fallback(P, dtype, static_cast<int>(ctas), stream);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return ENTMAX_ATTN_OK;
}

}  // namespace

namespace {

// FP8 screen sections: [q8 | q statistics | k8 | key-tile statistics | lists | counts].
struct ScreenView {
  void* q8;
  void* qst;
  void* k8;
  void* kst;
  int* list;
  int* count;
  size_t bytes;
};

ScreenView screen_view(void* base, const Layout& L, int B, int Hq, int Hkv, int T, bool packed) {
  ScreenView v;
  char* p = static_cast<char*>(base);
  const size_t nb = packed ? 1 : static_cast<size_t>(B);
  const size_t qrows = nb * Hq * T, krows = nb * Hkv * T, ktiles = nb * Hkv * L.slots;
  size_t off = 0;
  v.q8 = p + off;
  off += align256(qrows * 128);
  v.qst = p + off;
  off += align256(qrows * 16);
  v.k8 = p + off;
  off += align256(krows * 128);
  v.kst = p + off;
  off += align256(ktiles * 16);
  v.list = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * static_cast<size_t>(L.tiles) * L.nkt_max);
  v.count = reinterpret_cast<int*>(p + off);
  off += align256(sizeof(int) * static_cast<size_t>(L.tiles));
  v.bytes = off;
  return v;
}

}  // namespace

extern "C" {

int entmax_attn_tau_pass(const void* q, const void* k, float* tau, uint32_t* block_mask,
                         void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int T,
                         int d, float alpha, int n_iter, int causal, const int32_t* cu_seqlens,
                         int dtype, unsigned flags, cudaStream_t stream) {
  return tau_pass_impl(q, k, tau, block_mask, workspace, workspace_bytes, B, Hq, Hkv, T, d, alpha,
                       n_iter, causal, cu_seqlens, dtype, flags, stream);
}

size_t entmax_attn_screen_bytes(int B, int Hq, int Hkv, int T, int has_cu_seqlens) {
  Layout L;
  if (Hkv < 1 || Hq % Hkv != 0 || !make_layout(B, Hq, T, has_cu_seqlens != 0, &L)) return 0;
  return screen_view(nullptr, L, B, Hq, Hkv, T, has_cu_seqlens != 0).bytes;
}

int entmax_attn_tau_pass_screened(const void* q, const void* k, float* tau, uint32_t* block_mask,
                                  void* workspace, size_t workspace_bytes, void* screen,
                                  size_t screen_bytes, int B, int Hq, int Hkv, int T, int d,
                                  float alpha, int n_iter, int causal, const int32_t* cu_seqlens,
                                  int dtype, unsigned flags, cudaStream_t stream) {
  Layout L;
  ea::Problem P;
  int rc = check_and_describe(q, k, B, Hq, Hkv, T, d, alpha, n_iter, causal, cu_seqlens, dtype,
                              &L, &P);
  if (rc != ENTMAX_ATTN_OK) return rc;
  if (dtype != ENTMAX_ATTN_BF16 || d != 128 || !use_tensor_cores(dtype, flags) || !screen)
    return ENTMAX_ATTN_EINVAL;  // the screen runs on the tensor cores, bf16, d = 128
  if (reinterpret_cast<uintptr_t>(screen) & 255u) return ENTMAX_ATTN_EALIGN;
  const ScreenView sv = screen_view(screen, L, B, Hq, Hkv, T, cu_seqlens != nullptr);
  if (screen_bytes < sv.bytes) return ENTMAX_ATTN_ENOMEM;
  int err = ENTMAX_ATTN_OK;
  P.status = status_ptr(&err);
  if (!P.status) return err;
  cudaError_t e = ea::launch_screen(P, sv.q8, sv.qst, sv.k8, sv.kst, sv.list, sv.count, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return tau_pass_impl(q, k, tau, block_mask, workspace, workspace_bytes, B, Hq, Hkv, T, d, alpha,
                       n_iter, causal, cu_seqlens, dtype, flags, stream, sv.list, sv.count);
}

int entmax_attn_out_pass(const void* q, const void* k, const void* v, const float* tau,
                         const void* workspace, size_t workspace_bytes, void* out, int B, int Hq,
                         int Hkv, int T, int d, float alpha, int causal,
                         const int32_t* cu_seqlens, int dtype, unsigned flags,
                         cudaStream_t stream) {
  Layout L;
  ea::Problem P;
  int rc = check_and_describe(q, k, B, Hq, Hkv, T, d, alpha, 1, causal, cu_seqlens, dtype, &L,
                              &P);
  if (rc != ENTMAX_ATTN_OK) return rc;
  if (!v || !tau || !out || !workspace) return ENTMAX_ATTN_EINVAL;
  if (!aligned16(v) || !aligned16(tau) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ENTMAX_ATTN_EALIGN;
  const WsView wv = ws_view(const_cast<void*>(workspace), L);
  if (workspace_bytes < wv.min_bytes) return ENTMAX_ATTN_ENOMEM;
  int err = ENTMAX_ATTN_OK;
  P.status = status_ptr(&err);
  if (!P.status) return err;
  P.v = v;
  P.out = out;
  P.tau = const_cast<float*>(tau);
  attach_workspace(&P, wv);
  P.no_mask = (flags & ENTMAX_ATTN_FLAG_NO_BLOCK_MASK) ? 1 : 0;
  // with the support sections (the tau pass recorded into them), the recorded query tiles from
  // their lists and the tile pass for the pending ones; without, the tile pass for all
  P.from_support =
      ((flags & ENTMAX_ATTN_FLAG_SUPPORT) && workspace_bytes >= wv.bytes) ? 1 : 0;
  if ((flags & ENTMAX_ATTN_FLAG_OUT_FP32) && !use_tensor_cores(dtype, flags))
    return ENTMAX_ATTN_EINVAL;  // fp32 outputs of bf16 inputs: the tensor-core path only
  P.out_f32 = (flags & ENTMAX_ATTN_FLAG_OUT_FP32) ? 1 : 0;
  cudaError_t e = cudaSuccess;
  // only the tensor-core tau pass records supports; the CUDA-core path left every tile pending
  if (P.from_support && use_tensor_cores(dtype, flags)) e = ea::launch_out_support(P, stream);
  if (e == cudaSuccess)
    e = use_tensor_cores(dtype, flags) ? ea::launch_out_tc(P, stream)
                                       : ea::launch_out_simt(P, dtype, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ENTMAX_ATTN_OK;
}

int entmax_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* tau, const void* workspace, size_t workspace_bytes,
                    float* delta, float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int T,
                    int d, float alpha, int causal, const int32_t* cu_seqlens, int dtype,
                    unsigned flags, cudaStream_t stream) {
  Layout L;
  ea::Problem P;
  int rc = check_and_describe(q, k, B, Hq, Hkv, T, d, alpha, 1, causal, cu_seqlens, dtype, &L,
                              &P);
  if (rc != ENTMAX_ATTN_OK) return rc;
  if (!v || !dout || !tau || !workspace || !delta || !dq || !dk || !dv) return ENTMAX_ATTN_EINVAL;
  if (!aligned16(v) || !aligned16(dout) || !aligned16(tau) || !aligned16(delta) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ENTMAX_ATTN_EALIGN;
  const WsView wv = ws_view(const_cast<void*>(workspace), L);
  if (workspace_bytes < wv.min_bytes) return ENTMAX_ATTN_ENOMEM;
  int err = ENTMAX_ATTN_OK;
  P.status = status_ptr(&err);
  if (!P.status) return err;
  P.v = v;
  P.tau = const_cast<float*>(tau);
  attach_workspace(&P, wv);
  P.no_mask = (flags & ENTMAX_ATTN_FLAG_NO_BLOCK_MASK) ? 1 : 0;
  P.from_support =
      ((flags & ENTMAX_ATTN_FLAG_SUPPORT) && workspace_bytes >= wv.bytes) ? 1 : 0;
  const size_t kv_bytes = sizeof(float) * static_cast<size_t>(cu_seqlens ? 1 : B) * Hkv * T * d;
  cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, stream);
  if (e == cudaSuccess) e = ea::launch_bwd(P, dtype, dout, delta, dq, dk, dv, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ENTMAX_ATTN_OK;
}

namespace {

// Both passes on the library's cached workspace of (device, stream); flags as the two-pass form.
int fwd_cached(const void* q, const void* k, const void* v, void* out, float* tau,
               uint32_t* block_mask, int B, int Hq, int Hkv, int T, int d, float alpha,
               int n_iter, int causal, const int32_t* cu_seqlens, int dtype, unsigned flags,
               cudaStream_t stream) {
  Layout L;
  ea::Problem P;
  int rc = check_and_describe(q, k, B, Hq, Hkv, T, d, alpha, n_iter, causal, cu_seqlens, dtype,
                              &L, &P);
  if (rc != ENTMAX_ATTN_OK) return rc;
  if (!v || !out || !tau) return ENTMAX_ATTN_EINVAL;
  const size_t need = ws_view(nullptr, L).bytes;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(g_ws_mu);  // held until both passes are enqueued
  CachedWs& c = g_ws[{dev, stream}];
  if (c.bytes < need) {
    if (c.ptr) {
      e = cudaFreeAsync(c.ptr, stream);
      c.ptr = nullptr;
      c.bytes = 0;
      if (e != cudaSuccess) return cuda_fail(e);
    }
    e = cudaMallocAsync(&c.ptr, need, stream);
    if (e != cudaSuccess) {
      c.ptr = nullptr;
      cuda_fail(e);
      return ENTMAX_ATTN_ENOMEM;
    }
    c.bytes = need;
  }
  if (flags & ENTMAX_ATTN_FLAG_NO_BLOCK_MASK) {  // the pages' variant: the full output pass
    rc = entmax_attn_tau_pass(q, k, tau, block_mask, c.ptr, need, B, Hq, Hkv, T, d, alpha,
                              n_iter, causal, cu_seqlens, dtype, flags, stream);
    if (rc != ENTMAX_ATTN_OK) return rc;
    return entmax_attn_out_pass(q, k, v, tau, c.ptr, need, out, B, Hq, Hkv, T, d, alpha, causal,
                                cu_seqlens, dtype, flags, stream);
  }
  flags |= ENTMAX_ATTN_FLAG_SUPPORT;
  rc = entmax_attn_tau_pass(q, k, tau, block_mask, c.ptr, need, B, Hq, Hkv, T, d, alpha, n_iter,
                            causal, cu_seqlens, dtype, flags, stream);
  if (rc != ENTMAX_ATTN_OK) return rc;
  return entmax_attn_out_pass(q, k, v, tau, c.ptr, need, out, B, Hq, Hkv, T, d, alpha, causal,
                              cu_seqlens, dtype, flags, stream);
}

}  // namespace

int entmax_attn_rows(const void* x, long long ldx, void* p, long long ldp, float* tau, int rows,
                     int n, float alpha, int n_iter, int dtype, cudaStream_t stream) {
  if (!x || !p || rows < 1 || n < 1 || ldx < n || ldp < n || !(alpha > 1.f) ||
      !std::isfinite(alpha) ||
      n_iter < 1 || (dtype != ENTMAX_ATTN_FP32 && dtype != ENTMAX_ATTN_BF16))
    return ENTMAX_ATTN_EINVAL;
  const uintptr_t esz = dtype == ENTMAX_ATTN_FP32 ? 4u : 2u;
  if ((reinterpret_cast<uintptr_t>(x) % esz) || (reinterpret_cast<uintptr_t>(p) % esz) ||
      (reinterpret_cast<uintptr_t>(tau) & 3u))
    return ENTMAX_ATTN_EALIGN;
  cudaError_t e = ea::launch_entmax_rows(x, static_cast<int64_t>(ldx), p,
                                         static_cast<int64_t>(ldp), tau, rows, n, alpha, n_iter,
                                         dtype, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ENTMAX_ATTN_OK;
}

int entmax_attn_route_chunks(const void* q, const void* summaries, float* pi, float* tau, int B,
                             int Hq, int Hkv, int T, int d, int chunk_size, float alpha,
                             int n_iter, int causal, int estimate_diagonal, float scaling_factor,
                             int dtype, cudaStream_t stream) {
  if (!q || !summaries || !pi || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv != 0 ||
      B > 65535 || Hq > 65535 ||  // the search kernel's grid: (row blocks, heads, batches)
      d < 1 || d > 1024 || chunk_size < 1 || !std::isfinite(alpha) || !(alpha > 1.f) ||
      n_iter < 1 || n_iter > 1000 || (causal != 0 && causal != 1) ||
      (estimate_diagonal != 0 && estimate_diagonal != 1) || !std::isfinite(scaling_factor) ||
      (dtype != ENTMAX_ATTN_FP32 && dtype != ENTMAX_ATTN_BF16))
    return ENTMAX_ATTN_EINVAL;
  const int nc = (T - 1) / chunk_size + 1;
  const uintptr_t esz = dtype == ENTMAX_ATTN_FP32 ? 4u : 2u;
  if ((reinterpret_cast<uintptr_t>(q) % esz) || (reinterpret_cast<uintptr_t>(summaries) % esz) ||
      (reinterpret_cast<uintptr_t>(pi) & 3u) || (reinterpret_cast<uintptr_t>(tau) & 3u))
    return ENTMAX_ATTN_EALIGN;
  // the scores on the tensor cores where the shapes allow (bf16, d = 64 or 128, TMA-aligned
  // inputs, row counts within the tensor map's 32-bit coordinates), then the search
  const int64_t q_rows = static_cast<int64_t>(B) * Hq * T;
  const bool tc = dtype == ENTMAX_ATTN_BF16 && (d == 64 || d == 128) && aligned16(q) &&
                  aligned16(summaries) && q_rows < (int64_t(1) << 31) &&
                  static_cast<int64_t>(B) * Hkv * nc < (int64_t(1) << 31);
  cudaError_t e = cudaSuccess;
  if (tc) {
    int err = ENTMAX_ATTN_OK;
    int* st = status_ptr(&err);
    if (!st) return err;
    // the CUDA-core search kernel's own z scale, computed the same way
    const float zscale = (alpha - 1.f) * scaling_factor / sqrtf(static_cast<float>(d));
    e = ea::launch_route_scores_tc(q, summaries, pi, B, Hq, Hkv, T, d, nc, zscale, st, stream);
  }
  if (e == cudaSuccess)
    e = ea::launch_route_chunks(q, summaries, pi, tau, B, Hq, Hkv, T, d, nc, chunk_size, alpha,
                                n_iter, causal, estimate_diagonal, scaling_factor, dtype,
                                tc ? 1 : 0, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return ENTMAX_ATTN_OK;
}

int entmax_attn_fwd(const void* q, const void* k, const void* v, void* out, float* tau,
                    uint32_t* block_mask, int B, int Hq, int Hkv, int T, int d, float alpha,
                    int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                    cudaStream_t stream) {
  if (!block_mask) return ENTMAX_ATTN_EINVAL;
  return fwd_cached(q, k, v, out, tau, block_mask, B, Hq, Hkv, T, d, alpha, n_iter, causal,
                    cu_seqlens, dtype, 0u, stream);
}

int entmax_attn_fwd_no_block_mask(const void* q, const void* k, const void* v, void* out,
                                  float* tau, int B, int Hq, int Hkv, int T, int d, float alpha,
                                  int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                                  cudaStream_t stream) {
  return fwd_cached(q, k, v, out, tau, nullptr, B, Hq, Hkv, T, d, alpha, n_iter, causal,
                    cu_seqlens, dtype, ENTMAX_ATTN_FLAG_NO_BLOCK_MASK, stream);
}

int entmax_attn_fallback_tiles(const void* workspace, cudaStream_t stream) {
  if (!workspace) return -1;
  int n = 0;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemcpy(&n, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    cuda_fail(e);
    return -1;
  }
  return n;
}

int entmax_attn_status(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_entmax_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_entmax_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  return v;
}

void entmax_attn_release_workspaces(void) {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ws) {
    if (!kv.second.ptr) continue;
    cudaSetDevice(kv.first.first);
    cudaDeviceSynchronize();
    cudaFree(kv.second.ptr);
  }
  g_ws.clear();
  cudaSetDevice(cur);
}

const char* entmax_attn_strerror(int code) {
  switch (code) {
    case ENTMAX_ATTN_OK: return "ok";
    case ENTMAX_ATTN_EINVAL: return "invalid argument";
    case ENTMAX_ATTN_EALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case ENTMAX_ATTN_ECUDA: return "CUDA runtime error";
    case ENTMAX_ATTN_ETIMEOUT: return "device-side bounded wait timed out";
    case ENTMAX_ATTN_ENOMEM: return "workspace too small or allocation failed";
    default: return "unknown error code";
  }
}

const char* entmax_attn_last_cuda_error(void) { return g_cuda_err; }

}  // extern "C"
