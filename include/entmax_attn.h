/*
 * entmax_attn.h -- C ABI of the B200 (sm_100a) forward pass of causal alpha-entmax attention
 * with adaptive block skipping.
 *
 * The operation (AdaSplash: Adaptive Sparse Flash Attention, section "AdaSplash with Block
 * Masking"; alpha and causality as in its "Adaptive Sparsity Control" and "Causal and
 * Non-causal Masking" sections; packed batches as in "Variable Length Sequences"; grouped kv
 * heads as the enable_gqa option of the MiniCPM-4-8B-NSA page's "Usage" section):
 *
 *   s_ij = q_i . k_j / sqrt(d)                  k, v of kv head floor(h / (Hq / Hkv))
 *   p_ij = [(alpha - 1) s_ij - tau_i]_+ ^ (1 / (alpha - 1)),  tau_i such that sum_j p_ij = 1
 *   o_i  = sum_j p_ij v_j                          (p is used as computed; no renormalisation)
 *
 * over the valid keys j of row i: j <= i within the row's own sequence when causal, the whole
 * sequence otherwise.  tau_i is found by n_iter steps of a bracketed Halley + bisection search
 * ("Triton Entmax (Optimized Entmax Activation)" section of the same page).  The block mask
 * holds one bit per (128-row query tile, 128-key key tile): set iff some valid pair of the tile
 * has p > 0 (the per-block binary mask of the "AdaSplash with Block Masking" section, whose
 * memory grows with the product of the query-tile and key-tile counts).  The output pass
 * visits only the key tiles whose bit is set.
 *
 * Conventions for every entry point below:
 *   - Pointers named q, k, v, out, tau, block_mask, cu_seqlens, workspace are DEVICE pointers
 *     on the current CUDA device, owned by the caller, 16-byte aligned.  q, k, v, cu_seqlens
 *     are only read.
 *   - Layout, fixed length (cu_seqlens == NULL): q and out [B, Hq, T, d], k and v [B, Hkv, T, d],
 *     tau [B, Hq, T], all contiguous, row-major.
 *     Packed variable length (cu_seqlens != NULL): B is the number of sequences and T the total
 *     token count; q and out [Hq, T, d], k and v [Hkv, T, d], tau [Hq, T]; cu_seqlens int32
 *     [B + 1] with cu_seqlens[0] = 0, nondecreasing, cu_seqlens[B] = T.  cu_seqlens is read on
 *     the device only (no host synchronisation).  Attention never crosses sequences.
 *   - dtype: ENTMAX_ATTN_FP32 (q, k, v, out are float) or ENTMAX_ATTN_BF16 (bfloat16).  Scores
 *     and p are computed in fp32; BF16 products run on the tensor cores, FP32 ones on the CUDA
 *     cores in true fp32.
 *   - d must be 64 or 128; 1 < alpha, finite; n_iter >= 1; B, Hq, Hkv, T >= 1; Hq % Hkv == 0.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).  Errors found on the
 *     host are returned at once and nothing is launched; errors found on the device (a bounded
 *     wait that gave up) are latched in a per-device status word read by entmax_attn_status().
 *     No error is sticky: the next call starts clean.
 *
 * Block-mask layout (uint32 words, bit (kt & 31) of word (kt >> 5) stands for key tile kt,
 * key tiles counted from the start of the row's sequence):
 *   fixed length: [B, Hq, nQt, W] with nQt = ceil(T / 128) query tiles per head and
 *                 W = ceil(nQt / 32) words per query tile.
 *   packed:       [Hq, S, W] with S = floor(T / 128) + B query-tile slots per head and
 *                 W = ceil(ceil(T / 128) / 32).  Sequence b owns the slots starting at
 *                 floor(cu_seqlens[b] / 128) + b, one per query tile of the sequence, in order;
 *                 every other slot is all-zero.
 *   Every word is written; bits outside a tile's valid key range are zero.
 */
#ifndef ENTMAX_ATTN_H_
#define ENTMAX_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define ENTMAX_ATTN_OK 0
#define ENTMAX_ATTN_EINVAL 1   /* an argument is out of range or inconsistent */
#define ENTMAX_ATTN_EALIGN 2   /* a pointer is not 16-byte aligned */
#define ENTMAX_ATTN_ECUDA 3    /* a CUDA runtime call failed (see entmax_attn_last_cuda_error) */
#define ENTMAX_ATTN_ETIMEOUT 4 /* a device-side bounded wait gave up (status word) */
#define ENTMAX_ATTN_ENOMEM 5   /* workspace too small, or the library's allocation failed */

/* dtype codes. */
#define ENTMAX_ATTN_FP32 0
#define ENTMAX_ATTN_BF16 1

/* flags of the two-pass entry points (0 = the normal path). */
#define ENTMAX_ATTN_FLAG_CUDA_CORES 1u    /* run BF16 products on the CUDA cores too */
#define ENTMAX_ATTN_FLAG_ALL_FALLBACK 2u  /* send every query tile through the multi-sweep tau
                                             search that handles candidate-buffer overflow */
#define ENTMAX_ATTN_FLAG_NO_BLOCK_MASK 8u /* the variant without block mask (AdaSplash page,
                                             "adasplash_no_block_mask"): the tau pass writes no
                                             mask and no tile lists (block_mask may be NULL), and
                                             the output pass visits every causally valid key tile.
                                             Give it to both passes. */
#define ENTMAX_ATTN_FLAG_SUPPORT 16u      /* output from the supports; give it to both passes.
                                             The tensor-core tau pass records each row's support
                                             (the keys with p > 0 and their p) in the workspace,
                                             from its candidate buffers or, for query tiles whose
                                             buffers overflowed, from an extra sweep of its
                                             overflow kernel; the output pass computes o of those
                                             tiles from the lists and runs the tile pass over
                                             the others only (supports beyond a tile's list, the
                                             CUDA-core path, a workspace below
                                             entmax_attn_workspace_bytes).
                                             The path entmax_attn_fwd takes.  Give the
                                             output pass (and entmax_attn_bwd) this flag only
                                             after a tau pass with it on the same workspace. */
#define ENTMAX_ATTN_FLAG_OUT_FP32 32u     /* bf16 inputs on the tensor-core path: out is float
                                             (fp32 accumulations stored without rounding to
                                             bf16), same layout.  Give it to both passes;
                                             ENTMAX_ATTN_EINVAL with fp32 inputs or
                                             ENTMAX_ATTN_FLAG_CUDA_CORES. */
#define ENTMAX_ATTN_FLAG_TEST_STALL 4u    /* test hook of the bounded waits: the tensor-core tau
                                             pass never requests its query tiles, so each of its
                                             CTAs gives up after one wait limit (about 2 s) and
                                             the pass ends with ENTMAX_ATTN_ETIMEOUT in the
                                             status word; its outputs are void.  Use it on a
                                             problem of a few query tiles only. */

/* Full forward pass: the tau pass (tau search, block mask, and the support of every row whose
 * candidates it held), then the output pass (o from the supports, and over the active key tiles
 * of the remaining query tiles): the two-pass form with ENTMAX_ATTN_FLAG_SUPPORT.  Writes out,
 * tau and every word of block_mask.  Scratch memory (compact tile lists, overflow queue, support
 * lists) is allocated by the library on first use per (device, stream) with cudaMallocAsync on
 * `stream`, grown when a larger problem arrives, and kept until entmax_attn_release_workspaces().
 * Returns ENTMAX_ATTN_OK or an error code. */
int entmax_attn_fwd(const void* q, const void* k, const void* v, void* out, float* tau,
                    uint32_t* block_mask, int B, int Hq, int Hkv, int T, int d, float alpha,
                    int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                    cudaStream_t stream);

/* Number of uint32 words block_mask must hold (layout above); 0 on bad sizes. */
size_t entmax_attn_mask_words(int B, int Hq, int T, int has_cu_seqlens);

/* Query tiles (or slots) per head and words per query tile of the mask layout above.
 * Returns ENTMAX_ATTN_OK or ENTMAX_ATTN_EINVAL. */
int entmax_attn_mask_layout(int B, int Hq, int T, int has_cu_seqlens, int* tiles_per_head,
                            int* words_per_tile);

/* The full forward pass without the block mask: tau search, then the output pass over every
 * causally valid key tile (the pages' "adasplash_no_block_mask" variant).  The same out and tau as
 * entmax_attn_fwd (key tiles whose p are all zero add nothing), no mask written, workspace
 * handled as in entmax_attn_fwd.  Returns ENTMAX_ATTN_OK or an error code. */
int entmax_attn_fwd_no_block_mask(const void* q, const void* k, const void* v, void* out,
                                  float* tau, int B, int Hq, int Hkv, int T, int d, float alpha,
                                  int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                                  cudaStream_t stream);

/* Two-pass form, for callers that own the scratch memory or time the passes apart.
 * workspace: device memory of at least entmax_attn_workspace_bytes(...) bytes, 256-byte
 * aligned, owned by the caller; the tau pass fills it and the output pass reads it, so both
 * must see the same workspace, sizes and cu_seqlens, in stream order.  Returns 0 on bad sizes. */
size_t entmax_attn_workspace_bytes(int B, int Hq, int T, int has_cu_seqlens);

/* The smallest workspace the passes accept: the lists, counts and overflow queue without the
 * tau pass's warm-up keys (the squared key norms and, per key group, the 128 keys of largest
 * norm of a few prefix ranges, whose scores start every query tile's candidate threshold).  A
 * workspace between this size and entmax_attn_workspace_bytes() gives the same results, with
 * the bf16 tau pass running without warm-up keys.  Returns 0 on bad sizes. */
size_t entmax_attn_workspace_min_bytes(int B, int Hq, int T, int has_cu_seqlens);

/* Tau pass: writes tau, every word of block_mask, and the compact list of active key tiles of
 * every query tile into the workspace (with ENTMAX_ATTN_FLAG_SUPPORT also the supports).
 * ENTMAX_ATTN_ENOMEM if workspace_bytes is below entmax_attn_workspace_min_bytes(). */
int entmax_attn_tau_pass(const void* q, const void* k, float* tau, uint32_t* block_mask,
                         void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int T,
                         int d, float alpha, int n_iter, int causal, const int32_t* cu_seqlens,
                         int dtype, unsigned flags, cudaStream_t stream);

/* FP8 screening of the tau pass (AdaSplash page, "AdaSplash with Block Masking": the pass needs
 * only the keys that can carry p > 0, z_ij > tau_i >= max_j z_ij - 1).  A first sweep scores every
 * causal key tile on the tensor cores from e4m3 copies of q (one scale per row) and k (one scale
 * per 128-key tile) and bounds each score's error rigorously (Cauchy-Schwarz on the quantisation
 * errors, plus the accumulation); a key tile in which no row can reach its running lower bound
 * of the row max minus 1 (z units) holds no candidate and not the row max.  The bf16 tau pass
 * then scores only the other key tiles.  The results are those of entmax_attn_tau_pass (same
 * flags, workspace and outputs; give the output pass the same flags).  bf16 inputs on the tensor
 * cores with d = 128 only (ENTMAX_ATTN_EINVAL otherwise).  screen: device memory of at least
 * entmax_attn_screen_bytes(...) bytes, 256-byte aligned, owned by the caller (e4m3 copies of q
 * and k, their statistics, per query tile the screened key tiles); ENTMAX_ATTN_ENOMEM if smaller.
 * It costs one fp8 product per causal tile (half the tensor time of a bf16 one) and a bound test
 * per row and key tile, so it pays only where the screen removes more than half of the tiles. */
size_t entmax_attn_screen_bytes(int B, int Hq, int Hkv, int T, int has_cu_seqlens);
int entmax_attn_tau_pass_screened(const void* q, const void* k, float* tau, uint32_t* block_mask,
                                  void* workspace, size_t workspace_bytes, void* screen,
                                  size_t screen_bytes, int B, int Hq, int Hkv, int T, int d,
                                  float alpha, int n_iter, int causal, const int32_t* cu_seqlens,
                                  int dtype, unsigned flags, cudaStream_t stream);

/* Output pass: o_i = sum over the listed key tiles of p_ij v_j, with p recomputed from tau
 * (scores on the tensor cores, P rounded to bf16 for the P V product, fp32 accumulation).  With
 * ENTMAX_ATTN_FLAG_SUPPORT (given to the tau pass too): o_i = sum of p_ij v_j over the support
 * the tau pass recorded for row i (p in fp32 from the tau pass's own scores, fp32 accumulation,
 * one rounding to the output dtype), and the tile pass only for the query tiles without a
 * recorded support (AdaSplash page, "AdaSplash with Block Masking": p_ij > 0 needs
 * z_ij > tau_i >= max_j z_ij - 1, the keys the tau pass keeps to find tau). */
int entmax_attn_out_pass(const void* q, const void* k, const void* v, const float* tau,
                         const void* workspace, size_t workspace_bytes, void* out, int B, int Hq,
                         int Hkv, int T, int d, float alpha, int causal,
                         const int32_t* cu_seqlens, int dtype, unsigned flags,
                         cudaStream_t stream);

/* Backward pass: gradients of L = sum(dout * out) with respect to q, k and v, for the forward
 * pass whose tau and workspace (compact lists of active key tiles) the caller passes: run the tau
 * pass first (or entmax_attn_two_pass-style tau + output passes) on the same q, k, sizes and
 * cu_seqlens.  The AdaSplash page ("AdaSplash with Block Masking") says the forward's block mask
 * serves the backward pass too; only listed key tiles are visited.  The gradient follows the
 * alpha-entmax Jacobian diag(w) - w w^T / sum(w), w = p^(2 - alpha) (Peters, Niculae & Martins
 * 2019, Proposition 2): per query row, u_j = dout . v_j, delta = sum w u / sum w,
 * ds_j = w_j (u_j - delta), dq = sum ds_j k_j / sqrt(d), dk_j += ds_j q / sqrt(d),
 * dv_j += p_j dout.
 *   dout:  the upstream gradient, the layout and dtype of q.
 *   delta: fp32 [rows of q] written with the per-row delta (scratch the caller owns).
 *   dq:    fp32, the layout of q, fully written.
 *   dk, dv: fp32, the layout of k / v, fully written (zeroed, then accumulated over the query
 *          heads of each group).
 * Computed on the CUDA cores in fp32 from the stored inputs.  flags: ENTMAX_ATTN_FLAG_NO_BLOCK_MASK
 * visits every causally valid key tile instead of the lists (for a tau pass run with that flag);
 * ENTMAX_ATTN_FLAG_SUPPORT (for a forward run with that flag on this workspace, bf16) computes
 * the gradients of every row with a recorded support from its support list alone, and visits
 * the listed key tiles only for the other query tiles.
 * Device pointers 16-byte aligned (workspace 256), asynchronous on `stream`.  Returns
 * ENTMAX_ATTN_OK, ENTMAX_ATTN_EINVAL (as the forward, or a null pointer), ENTMAX_ATTN_EALIGN,
 * ENTMAX_ATTN_ENOMEM (workspace below entmax_attn_workspace_min_bytes) or ENTMAX_ATTN_ECUDA. */
int entmax_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* tau, const void* workspace, size_t workspace_bytes,
                    float* delta, float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int T,
                    int d, float alpha, int causal, const int32_t* cu_seqlens, int dtype,
                    unsigned flags, cudaStream_t stream);

/* Number of query tiles that the last tau pass on this workspace sent through the multi-sweep
 * overflow path.  Synchronises `stream`.  Returns -1 on a CUDA error. */
int entmax_attn_fallback_tiles(const void* workspace, cudaStream_t stream);

/* Row-wise alpha-entmax (AdaSplash page, "Triton Entmax (Optimized Entmax Activation)"): for every
 * row x of the [rows, n] matrix at `x` (row stride `ldx` elements, ldx >= n),
 *   p = [(alpha - 1) x - tau]_+^(1/(alpha - 1)),  tau such that sum(p) = 1,
 * written to the [rows, n] matrix at `p` (row stride `ldp` >= n), tau found by n_iter steps
 * (fewer once it has settled) of the bracketed Halley + bisection search of the attention passes.
 * x and p have the same dtype (ENTMAX_ATTN_FP32 or ENTMAX_ATTN_BF16) and may not overlap; tau
 * (fp32 [rows]) may be NULL.  Device pointers, aligned to their element size; asynchronous on
 * `stream`.  Returns ENTMAX_ATTN_OK, ENTMAX_ATTN_EINVAL (rows or n < 1, ldx or ldp < n, alpha <= 1
 * or not finite, n_iter < 1, bad dtype, null x or p), ENTMAX_ATTN_EALIGN or ENTMAX_ATTN_ECUDA. */
int entmax_attn_rows(const void* x, long long ldx, void* p, long long ldp, float* tau, int rows,
                     int n, float alpha, int n_iter, int dtype, cudaStream_t stream);

/* Entmax block routing over chunk summaries (MiniCPM-4-8B-NSA page, DashAttention, "How it
 * works", stage 2).  Keys are cut into chunks of chunk_size tokens, nc = ceil(T / chunk_size);
 * `summaries` holds one vector per (batch, kv head, chunk), [B, Hkv, nc, d], built by the caller.
 * Every query row i of q [B, Hq, T, d] scores the chunks it may see,
 *   s_c = scaling_factor * q_i . summaries[b, kv(h), c] / sqrt(d),   kv(h) = floor(h / (Hq / Hkv)),
 * and routes by alpha-entmax over them: pi_c = [(alpha - 1) s_c - tau_i]_+^(1/(alpha - 1)) with
 * sum_c pi_c = 1, tau_i by n_iter steps (fewer once settled) of the search of the attention passes.
 * Visible chunks: causal -- those before the row's own chunk floor(i / chunk_size), and the own
 * chunk too when estimate_diagonal is 1; not causal -- all.  Output: pi fp32 [B, Hq, T, nc], zero
 * outside the visible chunks (the routing priors; their nonzeros are the sparse chunk support);
 * tau fp32 [B, Hq, T] (may be NULL), +inf for a row that sees no chunk (its pi is all zero).
 * q and summaries share the dtype (ENTMAX_ATTN_FP32 or ENTMAX_ATTN_BF16), d <= 1024.  Device
 * pointers, aligned to their element size (pi, tau to 4 bytes); asynchronous on `stream`.
 * Returns ENTMAX_ATTN_OK, ENTMAX_ATTN_EINVAL (a size < 1, B or Hq above 65535, Hq not a multiple
 * of Hkv, d > 1024, alpha <= 1 or not finite, n_iter outside [1, 1000], causal or
 * estimate_diagonal not 0/1,
 * scaling_factor not finite, bad dtype, null q, summaries or pi), ENTMAX_ATTN_EALIGN or
 * ENTMAX_ATTN_ECUDA. */
int entmax_attn_route_chunks(const void* q, const void* summaries, float* pi, float* tau, int B,
                             int Hq, int Hkv, int T, int d, int chunk_size, float alpha,
                             int n_iter, int causal, int estimate_diagonal, float scaling_factor,
                             int dtype, cudaStream_t stream);

/* Synchronises `stream`, returns the device status word of the current device
 * (ENTMAX_ATTN_OK or ENTMAX_ATTN_ETIMEOUT) and clears it. */
int entmax_attn_status(cudaStream_t stream);

/* Frees the workspaces entmax_attn_fwd cached (synchronises the device first). */
void entmax_attn_release_workspaces(void);

/* Allocation-free forward pass.  The paper has no counterpart: this is a service for callers
 * that cannot allocate device memory while they run -- code inside an allocator or memory-pool
 * callback, where a nested cudaMalloc would recurse or deadlock; runtimes that forbid
 * allocation after start-up to keep a fixed footprint; launch sequences replayed from a
 * recording, where a first-use allocation would be an unrecorded side effect.
 * Same arguments, outputs and semantics as entmax_attn_fwd, but the scratch memory lives in a
 * file-scope device array of ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES that every GPU loading the
 * library holds until the process exits; the call allocates and frees nothing.
 *   - Problems whose smallest scratch (entmax_attn_workspace_min_bytes) exceeds that size are
 *     rejected with ENTMAX_ATTN_ENOMEM before anything is launched; those whose full scratch
 *     (entmax_attn_workspace_bytes) exceeds it run without the tau pass's warm-up keys.
 *   - The first call on a device, with that device current, looks up the array's device
 *     address (cudaGetSymbolAddress) and caches it; make that first call before any stream
 *     capture.
 *   - All calls on a device share the array and it keeps the last call's contents (each call
 *     rewrites everything it reads); calls that overlap on the GPU race on it, so serialise them
 *     (one stream, or events). */
#define ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
int entmax_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* tau,
                            uint32_t* block_mask, int B, int Hq, int Hkv, int T, int d,
                            float alpha, int n_iter, int causal, const int32_t* cu_seqlens,
                            int dtype, cudaStream_t stream);

/* The forward pass of entmax_attn_fwd on inputs and outputs in HOST memory.  q, k, v, out,
 * tau, block_mask and cu_seqlens are host pointers with the layouts and sizes above (page-locked
 * memory, e.g. from cudaHostAlloc, lets the copies run asynchronously and at full speed;
 * pageable memory works but each copy then waits for the host).  Every (batch row, kv head)
 * group -- packed batches: every kv head over all sequences -- is an independent problem and a
 * contiguous run of every array, so the call cuts the problem into chunks of whole groups and
 * streams them through a device staging buffer of two chunk slots: the copy in of chunk c + 1,
 * the computation of chunk c (entmax_attn_fwd on `stream`) and the copy out of chunk c - 1
 * overlap, with one cudaMemcpyAsync per contiguous run on two copy streams of the library.
 * Asynchronous: the call returns once everything is enqueued, and every output is in host
 * memory when `stream` has completed the work enqueued so far; keep the host buffers alive and
 * unmodified until then.  The staging buffer, the device copy of cu_seqlens and the copy
 * streams are allocated on first use per device and kept until the process exits; the
 * forward's workspace is entmax_attn_fwd's.  Calls on one device share one pipeline and take
 * turns (each call waits on the device for the previous one).  cu_seqlens (host) is checked on
 * the host: cu_seqlens[0] == 0, nondecreasing, cu_seqlens[B] == T.  Returns ENTMAX_ATTN_OK,
 * ENTMAX_ATTN_EINVAL (as entmax_attn_fwd, or a null pointer), ENTMAX_ATTN_ENOMEM (the staging
 * buffer could not be allocated) or ENTMAX_ATTN_ECUDA. */
int entmax_attn_fwd_host(const void* q, const void* k, const void* v, void* out, float* tau,
                         uint32_t* block_mask, int B, int Hq, int Hkv, int T, int d, float alpha,
                         int n_iter, int causal, const int32_t* cu_seqlens, int dtype,
                         cudaStream_t stream);

/* Static text for a return code. */
const char* entmax_attn_strerror(int code);

/* Text of the CUDA error behind the last ENTMAX_ATTN_ECUDA of this thread ("" if none). */
const char* entmax_attn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAX_ATTN_H_ */
