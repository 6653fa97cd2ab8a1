/*
 * fa.h -- C ABI of the fused tiled attention library (libfa.so, sm_100a).
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(Q K^T * scale + mask) V
 *
 * in one fused, tiled pass with an online softmax (running row maximum and row sum, with the
 * partial output rescaled whenever the maximum grows), so the score matrix never reaches
 * device memory.  Sources for each piece of the operation:
 *   - the formula softmax(QK^T / sqrt(d_k)) V and the [batch, seq_len, num_heads, head_dim]
 *     layout: "FlashAttention on Ascend NPUs", sections on the attention formula and on
 *     calling the operator (output has the shape of Q);
 *   - tiling of Q/K/V into blocks and the online softmax that keeps only the current maximum
 *     and exp-sum per row: "Flash Attention on Ascend: three techniques", sections 1 and 2;
 *   - MHA/GQA/MQA: query head h reads KV head floor(h / (Hq/Hkv)), the mapping of an explicit
 *     repeat_interleave of K and V along the head axis, which this library never builds:
 *     "FlashAttention variants: GQA, MQA, sparse attention", section on expanding KV;
 *   - causal and sliding-window masks (each query sees its W nearest keys, itself included):
 *     same page, sliding-window section;
 *   - decode over an INT8 KV cache computed without decompressing it first: "Flash
 *     Attention on Ascend: three techniques", section 3 (KV compression);
 *   - a paged KV cache addressed through a block_table, with one length per sequence:
 *     "Sparse attention and MLA operators in ops-transformer", section 2.2, and the
 *     three-techniques page, version section (dynamic sequence length).
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller, contiguous, 16-byte
 *     aligned.  The library allocates no device memory in these calls.  Besides host-side
 *     state (resolved driver entry points and per-device kernel attributes) it holds two kinds
 *     of static device data, reserved when the module loads on a device: a 4-byte status word
 *     (see fa_device_status) and the FA_DECODE_INT8_NOALLOC_MAX_SCRATCH-byte scratch array of
 *     fa_decode_int8_noalloc, which every GPU that loads the library holds until exit, even if
 *     only other entry points are called there.
 *   - bf16 tensors are raw IEEE bfloat16 bit patterns; fp32 tensors are IEEE binary32.
 *   - Calls validate their arguments synchronously and enqueue their kernels asynchronously on
 *     `stream` (a cudaStream_t; NULL is the legacy default stream).  Errors that happen on the
 *     device surface at the caller's next synchronisation; fa_device_status() reports the
 *     library's own device-side failures (a bounded wait that gave up, an out-of-range index
 *     read from device memory).
 *   - Thread safety: calls may be made from several host threads.  Their only shared mutable
 *     state is the guarded one-time initialisation, the per-device status word, and the
 *     scratch array of fa_decode_int8_noalloc (see there: calls of that function that overlap
 *     on the GPU race on it).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, Hq % Hkv != 0, bad window, ... */
  FA_ERR_UNSUPPORTED = -2, /* head dimension other than 64 or 128 */
  FA_ERR_ALIGNMENT = -3,   /* a tensor pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = -4,   /* decode workspace missing or smaller than required */
  FA_ERR_CUDA = -5,        /* a CUDA runtime/driver call or a kernel launch failed */
  FA_ERR_TIMEOUT = -6,     /* a kernel gave up a bounded wait (reported by fa_device_status) */
  FA_ERR_DEVICE_INDEX = -7 /* a page id or sequence length read on the device was out of range
                              (reported by fa_device_status) */
} fa_status;

/*
 * Prefill / full forward pass.
 *   q    bf16 [B, Sq,  Hq,  D]
 *   k, v bf16 [B, Skv, Hkv, D]
 *   o    bf16 [B, Sq,  Hq,  D]   written; may not alias q, k or v
 *   lse  fp32 [B, Hq, Sq]        natural-log log-sum-exp of each row's scaled, masked scores,
 *                                or NULL to skip it.  A row that sees no key gets O = 0 and
 *                                LSE = -inf.
 *   scale   > 0 and finite (1/sqrt(D) for the usual attention).
 *   causal  0 or 1.  The causal mask is aligned to the bottom-right corner: query i sees key j
 *           iff j <= i + (Skv - Sq).
 *   window  <= 0: none.  > 0 (only with causal = 1): query i also needs j > i + (Skv - Sq) -
 *           window, i.e. it sees its `window` nearest keys including its own position.
 *   D must be 64 or 128; Hq must be a multiple of Hkv.
 * Returns FA_OK or an fa_status error code; nothing is launched on error.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Sq, int Skv, int D, float scale, int causal, int window, void* stream);

/*
 * Forward pass with an additive mask tensor and / or global tokens, on top of fa_fwd's causal
 * and window rule.  Sources: "FlashAttention variants: GQA, MQA, sparse attention",
 * sliding-window section (the mask given as atten_mask, -inf where a key is dropped) and
 * global+local section (a few global tokens attend to, and are attended by, every token).
 *   n_global  >= 0.  Query i sees key j when the causal / window rule admits it, or j <
 *             n_global, or i < n_global (global tokens are the first n_global positions of
 *             both the query and the key sequence).  Key tiles no query of a block needs are
 *             never loaded.
 *   mask      fp32 or NULL: element (b, h, i, j) at mask[b * mask_batch_stride + h *
 *             mask_head_stride + i * Skv + j], added to scale * q.k; -inf drops the key.  A zero
 *             stride broadcasts over batch or heads.  16-byte aligned; rows are read with vector
 *             loads when Skv and both strides are multiples of 4.
 * Every other argument is that of fa_fwd; fa_fwd(...) is fa_fwd_ext(..., 0, NULL, 0, 0, ...).
 * A row whose every key is dropped gets O = 0 and LSE = -inf.
 */
FA_API int fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal,
                      int window, int n_global, const float* mask, int64_t mask_batch_stride,
                      int64_t mask_head_stride, void* stream);

/*
 * Backward pass: gradients of sum(dout * O) with respect to q, k, v for O = fa_fwd(q, k, v) with
 * the same causal / window rule.  The probabilities are recomputed tile by tile from q, k and
 * the forward pass's log-sum-exp rather than stored ("FlashAttention on Ascend NPUs",
 * recomputation section).
 *   q, o, dout  bf16 [B, Sq, Hq, D]      (o and lse as returned by fa_fwd for these inputs)
 *   k, v        bf16 [B, Skv, Hkv, D]
 *   lse         fp32 [B, Hq, Sq], natural log (required)
 *   dq          bf16 [B, Sq, Hq, D]  written
 *   dk, dv      bf16 [B, Skv, Hkv, D] written; for GQA / MQA they sum over the query heads that
 *               read each KV head
 *   workspace   at least fa_bwd_workspace_bytes(B, Hq, Sq) bytes, 16-byte aligned: per-row
 *               D = dO . O and the log-sum-exp in log2 units, then an fp32 dQ accumulator
 *               [B, Sq, Hq, 128] (sized for D = 128 whatever D is); contents on entry do not
 *               matter.
 * Other arguments as for fa_fwd.  Three kernels run in order on `stream`: a per-row pass (D, L,
 * and the accumulator zeroed), one kernel per (b, KV head, 128-key tile) that writes dK and dV
 * and adds the tile's share of dQ into the accumulator (TMA tensor reductions), and a pass that
 * scales the accumulator and rounds it to bf16.  dK and dV are deterministic; dQ is a sum of
 * fp32 shares whose order depends on timing, so it can differ between runs in its last bits.
 * Returns FA_OK or an fa_status error code.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int Hq, int Sq);
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
                  int Skv, int D, float scale, int causal, int window, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace fa_decode_int8 needs: fp32 partial outputs [num_splits, B, Hq, D]
 * followed by fp32 partial log-sum-exps [num_splits, B, Hq], padded to 256 bytes.
 * Returns 0 for invalid sizes.
 */
FA_API size_t fa_decode_int8_workspace_bytes(int B, int Hq, int D, int num_splits);

/*
 * Decode step (one query token per sequence) over an INT8 KV cache, split over the keys.
 *   q       bf16 [B, 1, Hq, D]
 *   k, v    int8 [B, Skv, Hkv, D]   codes; element value = code * scale of its (token, head)
 *   k_scale, v_scale fp32 [B, Hkv, Skv]
 *   o       bf16 [B, 1, Hq, D]     written
 *   lse     fp32 [B, Hq] natural log, or NULL
 *   num_splits >= 1: the keys are cut into chunks of ceil(Skv / num_splits) keys rounded up to
 *           a multiple of 128 (so fewer chunks than num_splits may hold keys); each chunk is
 *           reduced to a partial (output, log-sum-exp) in `workspace`, and a second kernel
 *           merges the partials through their log-sum-exp.
 *   workspace  device buffer of at least fa_decode_int8_workspace_bytes(B, Hq, D, num_splits)
 *           bytes, owned by the caller; its contents on entry do not matter.  Two calls that may
 *           run concurrently must not share one workspace.
 * The query sees every key (causal alignment of a single query at the end of the sequence).
 * D must be 64 or 128; Hq must be a multiple of Hkv.
 */
FA_API int fa_decode_int8(const void* q, const int8_t* k, const int8_t* v, const float* k_scale,
                   const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Skv,
                   int D, float scale, int num_splits, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * Allocation-free variant of fa_decode_int8 (the pages have no counterpart; this is a calling
 * convenience of this library).
 *
 * Who needs it: callers that cannot call cudaMalloc at the point where they decode -- code
 * running under a memory manager that owns the whole device budget and forbids allocations it
 * did not make, latency-critical loops where an allocation's implicit device synchronisation is
 * not acceptable, and plain C callers without an allocator of their own.  They pass inputs and
 * outputs exactly as for fa_decode_int8 but no workspace.
 *
 * Scratch: the split partials live in a fixed array inside the library, of
 * FA_DECODE_INT8_NOALLOC_MAX_SCRATCH bytes per GPU, which every GPU that loads the library holds
 * until the process exits.  Calls whose fa_decode_int8_workspace_bytes(B, Hq, D, num_splits)
 * exceeds that size return FA_ERR_WORKSPACE and launch nothing.  This function calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current and caches it.  If no other fa_* call has launched a kernel on that device
 * yet, that lookup is also what loads the library's module there (CUDA loads modules lazily),
 * and loading the module reserves the array and the kernels' code: an implicit allocation that
 * may synchronise the device.  Callers for whom that matters make one call of this function (or
 * of any fa_* entry point that launches a kernel) on each device at set-up time, before any
 * stream capture and before the latency-critical or allocation-free part of their program.
 *
 * Every call on a GPU shares the one array, and the array keeps the last call's contents (the
 * kernels overwrite every byte they read, so nothing needs clearing).  Calls whose kernels can
 * overlap on the GPU -- on different streams, or from different host threads -- race on it;
 * order such calls on one stream or use fa_decode_int8 with separate workspaces.
 * Arguments, layouts and status codes are otherwise those of fa_decode_int8.
 */
#define FA_DECODE_INT8_NOALLOC_MAX_SCRATCH (8u << 20)
FA_API int fa_decode_int8_noalloc(const void* q, const int8_t* k, const int8_t* v,
                                  const float* k_scale, const float* v_scale, void* o, float* lse,
                                  int B, int Hq, int Hkv, int Skv, int D, float scale,
                                  int num_splits, void* stream);

/*
 * Decode step over a PAGED INT8 KV cache with one length per sequence.
 * Sources: the KV cache stored in pages that a block_table maps to each sequence ("Sparse
 * attention and MLA operators in ops-transformer", section 2.2, paged attention through a
 * block_table); sequences of different lengths computed in one batch ("Flash Attention on
 * Ascend: three techniques", version section, dynamic sequence length); the INT8 cache used
 * without decompressing it first (same page, section 3).
 *   q        bf16 [B, 1, Hq, D]
 *   k_pages, v_pages  int8 [num_pages, page_size, Hkv, D]   a pool of pages of page_size tokens
 *   k_scale_pages, v_scale_pages  fp32 [num_pages, Hkv, page_size]  one scale per (token, head)
 *   block_table  int32 [B, max_pages_per_seq] (device): key j of sequence b is row
 *            j % page_size of page block_table[b][j / page_size].  Entries past a sequence's
 *            last page are never read and may hold anything.
 *   seqlens  int32 [B] (device): number of keys of each sequence, 0 .. max_pages_per_seq *
 *            page_size.  A sequence with 0 keys gets O = 0 and LSE = -inf.
 *   o, lse   as for fa_decode_int8.
 *   page_size  a power of two, 16 .. 65536; max_pages_per_seq * page_size <= 2^30.
 *   num_pages  number of pages in the pool (page ids are 0 .. num_pages - 1).
 *   num_splits >= 1: each sequence's keys are cut into chunks of ceil(seqlens[b] / num_splits)
 *            keys rounded up to a multiple of 128 (a short sequence fills only its first
 *            chunks); chunks are merged through their log-sum-exp as in fa_decode_int8.
 *   workspace  at least fa_decode_int8_workspace_bytes(B, Hq, D, num_splits) bytes.
 * block_table and seqlens need 4-byte alignment; every other tensor 16-byte alignment.
 * The lengths and page ids live in device memory, so they are checked on the device: an id
 * outside 0 .. num_pages - 1 or a length outside the range above is replaced by a valid one (no
 * access ever leaves the pool) and recorded, and the next fa_device_status() returns
 * FA_ERR_DEVICE_INDEX; the outputs of that call are then undefined.
 * D must be 64 or 128; Hq must be a multiple of Hkv.  Returns FA_OK or an fa_status error code;
 * nothing is launched on error.
 */
FA_API int fa_decode_int8_paged(const void* q, const int8_t* k_pages, const int8_t* v_pages,
                                const float* k_scale_pages, const float* v_scale_pages,
                                const int32_t* block_table, const int32_t* seqlens, void* o,
                                float* lse, int B, int Hq, int Hkv, int page_size,
                                int max_pages_per_seq, int num_pages, int D, float scale,
                                int num_splits, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Decode step over an INT4 KV cache (the KV-compression section of "Flash Attention on Ascend:
 * three techniques" names INT4 beside INT8; the pages give no packing, this library's format
 * is the following).  Two codes per byte: byte i of a key row holds dim 2i in bits 0-3 and dim
 * 2i+1 in bits 4-7, each a 4-bit two's-complement code; element value = code * scale of its
 * (token, KV head).
 *   k, v    uint8 [B, Skv, Hkv, D/2]   packed codes
 *   every other argument, layout, status code and the split semantics are those of
 *   fa_decode_int8 (the workspace size is fa_decode_int8_workspace_bytes).
 */
FA_API int fa_decode_int4(const void* q, const uint8_t* k, const uint8_t* v, const float* k_scale,
                          const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv,
                          int Skv, int D, float scale, int num_splits, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * Paged, variable-length decode over an INT4 KV cache: fa_decode_int8_paged with
 * k_pages, v_pages uint8 [num_pages, page_size, Hkv, D/2] packed as for fa_decode_int4.
 */
FA_API int fa_decode_int4_paged(const void* q, const uint8_t* k_pages, const uint8_t* v_pages,
                                const float* k_scale_pages, const float* v_scale_pages,
                                const int32_t* block_table, const int32_t* seqlens, void* o,
                                float* lse, int B, int Hq, int Hkv, int page_size,
                                int max_pages_per_seq, int num_pages, int D, float scale,
                                int num_splits, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Static, human-readable name of a status code.  Never NULL. */
FA_API const char* fa_status_string(int status);

/*
 * Takes the library's device status word on the current device: a one-thread kernel on
 * `stream` swaps it with 0 in one atomic operation, so a bit that a running kernel sets is
 * never lost between the read and the clear; then `stream` is synchronised and the old value
 * read back.  Returns FA_ERR_TIMEOUT if a kernel launched by this library gave up a bounded wait
 * since the last call, else FA_ERR_DEVICE_INDEX if a kernel met an out-of-range page id or
 * sequence length (the outputs of such a call are undefined), FA_ERR_CUDA if a CUDA call
 * failed, else FA_OK.
 * The word is one per device and process, not per stream: it collects the reports of every
 * kernel of this library on that device, whatever stream launched it, and a call consumes
 * them all.  Callers that run several streams should call it after synchronising all of them.
 * Concurrent calls from several host threads are serialised by the library.
 */
FA_API int fa_device_status(void* stream);

/*
 * Diagnostic: launches one thread that waits on a shared-memory barrier nothing ever signals,
 * with a wall-clock limit of `timeout_us` microseconds (1 .. 10^7).  The wait gives up, records
 * the timeout in the device status word and the kernel returns normally, so a following
 * fa_device_status() returns FA_ERR_TIMEOUT.  This exercises the same bounded-wait code every
 * kernel of the library uses, without faulting or hanging the device.
 */
FA_API int fa_selftest_bounded_wait(int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
