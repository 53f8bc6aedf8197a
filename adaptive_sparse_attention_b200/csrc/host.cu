// host.cu -- entmax_attn_fwd_host: the forward pass on inputs and outputs in host memory,
// streamed through the GPU in chunks so that the copies in, the computation and the copies out
// overlap.
//
// Every (batch row, kv head) group -- its kv head's keys and values and the G query heads that
// read them -- is an independent problem, and in the documented layouts each group is one
// contiguous run of q, k, v, out, tau and the block mask (packed batches: each kv head's group
// spans all sequences).  The call cuts the problem into chunks of whole groups and runs, for
// chunk c, in slot c % 2 of a device staging buffer:
//   copy stream in:   q, k, v of chunk c (after chunk c - 2's computation has read the slot)
//   caller's stream:  entmax_attn_fwd on the slot (after the copy in, and after chunk c - 2's
//                     outputs have been copied out of the slot)
//   copy stream out:  out, tau and the mask words of chunk c
// so that with two chunks in flight the step takes about the longer of the two copy directions
// (PCIe moves both at once) plus one chunk's copy in and copy out.  Each copy is one
// cudaMemcpyAsync of a contiguous run.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <map>
#include <mutex>

#include "entmax_attn.h"
#include "kernels.h"

namespace {

constexpr int kSlots = 2;
constexpr int kTargetChunks = 16;  // more chunks: less unoverlapped copy at both ends

// Per device: the two copy streams, the events of the pipeline and the staging buffer.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kSlots] = {}, comp_done[kSlots] = {}, out_done[kSlots] = {};
  void* buf = nullptr;
  size_t bytes = 0;
  int32_t* cu = nullptr;
  size_t cu_bytes = 0;
};

std::mutex g_host_mu;
std::map<int, HostPipe> g_pipes;

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

cudaError_t pipe_init(HostPipe& p) {
  if (p.in) return cudaSuccess;
  cudaError_t e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.end, cudaEventDisableTiming);
  for (int s = 0; s < kSlots && e == cudaSuccess; ++s) {
    e = cudaEventCreateWithFlags(&p.in_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.comp_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.out_done[s], cudaEventDisableTiming);
  }
  return e;
}

// Grows a device buffer (stream-ordered free of the old one after everything the pipe issued).
cudaError_t ensure(void** ptr, size_t* have, size_t need, cudaStream_t s) {
  if (*have >= need) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (*ptr) e = cudaFreeAsync(*ptr, s);
  *ptr = nullptr;
  *have = 0;
  if (e != cudaSuccess) return e;
  e = cudaMallocAsync(ptr, need, s);
  if (e != cudaSuccess) {
    *ptr = nullptr;
    return e;
  }
  *have = need;
  return cudaSuccess;
}

}  // namespace

extern "C" int entmax_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                    float* tau, uint32_t* block_mask, int B, int Hq, int Hkv,
                                    int T, int d, float alpha, int n_iter, int causal,
                                    const int32_t* cu_seqlens, int dtype, cudaStream_t stream) {
  if (!q || !k || !v || !out || !tau || !block_mask) return ENTMAX_ATTN_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv != 0) return ENTMAX_ATTN_EINVAL;
  if (dtype != ENTMAX_ATTN_FP32 && dtype != ENTMAX_ATTN_BF16) return ENTMAX_ATTN_EINVAL;
  const bool packed = cu_seqlens != nullptr;
  if (packed) {  // the host holds cu_seqlens: check it here
    if (cu_seqlens[0] != 0 || cu_seqlens[B] != T) return ENTMAX_ATTN_EINVAL;
    for (int b = 0; b < B; ++b)
      if (cu_seqlens[b + 1] < cu_seqlens[b]) return ENTMAX_ATTN_EINVAL;
  }
  int slots = 0, W = 0;
  if (entmax_attn_mask_layout(B, Hq, T, packed ? 1 : 0, &slots, &W) != ENTMAX_ATTN_OK)
    return ENTMAX_ATTN_EINVAL;
  const int G = Hq / Hkv;
  const size_t esz = dtype == ENTMAX_ATTN_FP32 ? 4 : 2;
  // groups: (batch row, kv head) for fixed length, kv head for a packed batch; a chunk is n
  // consecutive kv heads of one batch row (n divides Hkv)
  const int rows_b = packed ? 1 : B;
  int n = std::max(1, (rows_b * Hkv + kTargetChunks - 1) / kTargetChunks);
  while (Hkv % n) ++n;
  const int per_row = Hkv / n, chunks = rows_b * per_row;
  const size_t kv_elems = static_cast<size_t>(n) * T * d;       // k (or v) of one chunk
  const size_t q_elems = kv_elems * G;                          // q (or out) of one chunk
  const size_t tau_elems = static_cast<size_t>(n) * G * T;
  const size_t mask_words = static_cast<size_t>(n) * G * slots * W;
  const size_t off_k = up256(q_elems * esz), off_v = off_k + up256(kv_elems * esz);
  const size_t off_o = off_v + up256(kv_elems * esz), off_t = off_o + up256(q_elems * esz);
  const size_t off_m = off_t + up256(tau_elems * 4), slot_bytes = off_m + up256(mask_words * 4);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ea::record_cuda_error(e);
  std::lock_guard<std::mutex> lk(g_host_mu);  // one pipeline per device: calls take turns
  HostPipe& p = g_pipes[dev];
  if ((e = pipe_init(p)) != cudaSuccess) return ea::record_cuda_error(e);
  // order: after the caller's earlier work on `stream` and after this pipe's previous call
  if ((e = cudaEventRecord(p.start, stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(p.in, p.start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(p.in, p.end, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(p.out, p.start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(stream, p.end, 0)) != cudaSuccess)
    return ea::record_cuda_error(e);
  if ((e = ensure(&p.buf, &p.bytes, kSlots * slot_bytes, stream)) != cudaSuccess) {
    ea::record_cuda_error(e);
    return ENTMAX_ATTN_ENOMEM;
  }
  const size_t cu_need = packed ? sizeof(int32_t) * (B + 1) : 0;
  if (packed) {
    void* cp = p.cu;
    e = ensure(&cp, &p.cu_bytes, cu_need, stream);
    p.cu = static_cast<int32_t*>(cp);
    if (e != cudaSuccess) {
      ea::record_cuda_error(e);
      return ENTMAX_ATTN_ENOMEM;
    }
  }
  // the copy stream waits for the allocations made on `stream`
  if ((e = cudaEventRecord(p.start, stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(p.in, p.start, 0)) != cudaSuccess)
    return ea::record_cuda_error(e);
  if (packed && (e = cudaMemcpyAsync(p.cu, cu_seqlens, cu_need, cudaMemcpyHostToDevice,
                                     p.in)) != cudaSuccess)
    return ea::record_cuda_error(e);

  const char* qh = static_cast<const char*>(q);
  const char* kh = static_cast<const char*>(k);
  const char* vh = static_cast<const char*>(v);
  char* oh = static_cast<char*>(out);
  char* th = reinterpret_cast<char*>(tau);
  char* mh = reinterpret_cast<char*>(block_mask);
  int rc = ENTMAX_ATTN_OK;
  for (int c = 0; c < chunks && rc == ENTMAX_ATTN_OK; ++c) {
    const int s = c % kSlots;
    char* base = static_cast<char*>(p.buf) + s * slot_bytes;
    const size_t i = static_cast<size_t>(c);  // chunk index = (batch row, kv-head range)
    // copy in (the slot's inputs are free once chunk c - 2's computation is done)
    if (c >= kSlots && (e = cudaStreamWaitEvent(p.in, p.comp_done[s], 0)) != cudaSuccess) break;
    if ((e = cudaMemcpyAsync(base, qh + i * q_elems * esz, q_elems * esz,
                             cudaMemcpyHostToDevice, p.in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(base + off_k, kh + i * kv_elems * esz, kv_elems * esz,
                             cudaMemcpyHostToDevice, p.in)) != cudaSuccess ||
        (e = cudaMemcpyAsync(base + off_v, vh + i * kv_elems * esz, kv_elems * esz,
                             cudaMemcpyHostToDevice, p.in)) != cudaSuccess ||
        (e = cudaEventRecord(p.in_done[s], p.in)) != cudaSuccess)
      break;
    // compute (its outputs are free once chunk c - 2's copy out is done)
    if ((e = cudaStreamWaitEvent(stream, p.in_done[s], 0)) != cudaSuccess) break;
    if (c >= kSlots && (e = cudaStreamWaitEvent(stream, p.out_done[s], 0)) != cudaSuccess) break;
    rc = entmax_attn_fwd(base, base + off_k, base + off_v, base + off_o,
                         reinterpret_cast<float*>(base + off_t),
                         reinterpret_cast<uint32_t*>(base + off_m), packed ? B : 1, n * G, n, T,
                         d, alpha, n_iter, causal, packed ? p.cu : nullptr, dtype, stream);
    if (rc != ENTMAX_ATTN_OK) break;
    if ((e = cudaEventRecord(p.comp_done[s], stream)) != cudaSuccess) break;
    // copy out
    if ((e = cudaStreamWaitEvent(p.out, p.comp_done[s], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(oh + i * q_elems * esz, base + off_o, q_elems * esz,
                             cudaMemcpyDeviceToHost, p.out)) != cudaSuccess ||
        (e = cudaMemcpyAsync(th + i * tau_elems * 4, base + off_t, tau_elems * 4,
                             cudaMemcpyDeviceToHost, p.out)) != cudaSuccess ||
        (e = cudaMemcpyAsync(mh + i * mask_words * 4, base + off_m, mask_words * 4,
                             cudaMemcpyDeviceToHost, p.out)) != cudaSuccess ||
        (e = cudaEventRecord(p.out_done[s], p.out)) != cudaSuccess)
      break;
  }
  // `stream` completes only after every copy out; the next call starts after this one
  cudaError_t e2 = cudaEventRecord(p.end, p.out);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(stream, p.end, 0);
  if (e == cudaSuccess) e = e2;
  if (e != cudaSuccess) return ea::record_cuda_error(e);
  return rc;
}
