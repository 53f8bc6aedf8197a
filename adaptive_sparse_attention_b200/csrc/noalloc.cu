// noalloc.cu -- entmax_attn_fwd_noalloc: the full forward pass with its scratch memory in a
// fixed device array instead of memory obtained from cudaMalloc.
//
// Who needs it: code that must not allocate device memory while it runs -- a caller inside a
// custom allocator or memory-pool callback (where a nested cudaMalloc would recurse or
// deadlock), a runtime that forbids allocation after start-up so that its footprint stays
// fixed, or one that replays launches from a recorded sequence in which a first-use allocation
// would be an unrecorded side effect.  entmax_attn_fwd allocates its workspace on first use;
// this entry point never does.
//
// The scratch is g_noalloc_scratch below: ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES (16 MiB) of device
// memory, present on every GPU that loads the library until the process exits.  In host code
// the array's name is only a host-side stand-in, so its device address is fetched with
// cudaGetSymbolAddress, once per device, on the first call made with that device current.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "entmax_attn.h"
#include "kernels.h"

namespace {

// Scratch of every call of entmax_attn_fwd_noalloc on this device.  Calls share it: each call
// overwrites what it needs (the tau pass clears the overflow counter and writes every list and
// count that the output pass then reads), and calls that overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

}  // namespace

extern "C" int entmax_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                       float* tau, uint32_t* block_mask, int B, int Hq, int Hkv,
                                       int T, int d, float alpha, int n_iter, int causal,
                                       const int32_t* cu_seqlens, int dtype,
                                       cudaStream_t stream) {
  const size_t need = entmax_attn_workspace_min_bytes(B, Hq, T, cu_seqlens != nullptr);
  if (need == 0) return ENTMAX_ATTN_EINVAL;
  if (need > ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES) return ENTMAX_ATTN_ENOMEM;  // too large for it

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ea::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return ea::record_cuda_error(cudaErrorInvalidDevice);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return ea::record_cuda_error(e);
      if (p == nullptr) return ea::record_cuda_error(cudaErrorInvalidSymbol);
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  int rc = entmax_attn_tau_pass(q, k, tau, block_mask, scratch, ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES,
                                B, Hq, Hkv, T, d, alpha, n_iter, causal, cu_seqlens, dtype,
                                ENTMAX_ATTN_FLAG_SUPPORT, stream);
  if (rc != ENTMAX_ATTN_OK) return rc;
  return entmax_attn_out_pass(q, k, v, tau, scratch, ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES, out, B,
                              Hq, Hkv, T, d, alpha, causal, cu_seqlens, dtype,
                              ENTMAX_ATTN_FLAG_SUPPORT, stream);
}
