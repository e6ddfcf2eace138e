/*
 * frt_attn.h -- C ABI of the B200 (sm_100a) fused-attention library.
 *
 * Three operations, each the FlashAttention-style computation of softmax
 * attention that the pages describe:
 *   - "Real-time inference optimisation: making large models respond fast"
 *     (llmapi-app.pages.dev), section "Flash Attention optimisation": tiled
 *     Q.K^T times a scale, online softmax (running max and sum, rescaling the
 *     accumulator), P.V accumulation, final division by the sum; method
 *     paged_attention: a KV cache in pages of 16 tokens.
 *   - "FlashRT-HF-kernels" (zingnex.cn), section "Attention optimisation":
 *     blockwise computation without storing the attention matrix, causal
 *     masking for autoregressive generation, MQA/GQA; section "Attention
 *     operators": flash attention, cross attention, paged attention.
 *   - "Analysis of TensorRT's low-level support for FlashAttention"
 *     (yongjin360.com), the plugin
 *     sketch: the kernel is launched on the caller's stream with Q, K, V, O,
 *     head count, query and key lengths and head dimension, and returns 0.
 *
 * Definition computed (all three calls).  For batch b, query head h, query i,
 * with g = Hq / Hkv and KV head kvh = h / g:
 *   s_ij = scale * sum_d q[b,h,i,d] * k[b,kvh,j,d]
 *   key j is visible to query i iff  !causal || j <= i + (Skv - Sq)
 *   o[b,h,i,:] = sum_j softmax_j(s_ij) * v[b,kvh,j,:]   over visible j
 *   lse[b,h,i] = log(sum_j exp(s_ij))                    natural log, scale included
 * A row with no visible key gets o = 0 and lse = -inf.  The causal mask is
 * aligned bottom-right (the last query sees every key), which is the usual
 * lower-triangular mask when Sq == Skv; the pages do not fix the alignment
 * for Sq != Skv, this is the library's reading.
 *
 * Conventions shared by every call:
 *   - All pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or synchronises.  Every call is asynchronous on
 *     `stream`; a device-side failure (an internal wait that timed out) is
 *     reported by frt_read_device_error(), never by a hang.
 *   - Tensors are contiguous, row-major, with the shapes given; q/k/v/o are
 *     bf16 (uint16 bit patterns), lse is fp32.  Every pointer must be 16-byte
 *     aligned.  Head dimension D is 64 or 128.
 *   - Arguments are validated before anything is launched; a rejected call
 *     returns a non-zero status and leaves every output untouched.
 *   - Arithmetic: bf16 inputs, fp32 accumulation, exp2-based softmax with
 *     the scale folded into the exponent, P rounded to bf16 before the P.V
 *     product, O rounded once to bf16 (round to nearest even).
 */
#ifndef FRT_ATTN_H_
#define FRT_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FRT_API __attribute__((visibility("default")))
#else
#define FRT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FRT_OK = 0,
  FRT_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, Hq % Hkv != 0, bad scale */
  FRT_ERR_UNSUPPORTED = 2,   /* valid but not implemented here (e.g. D not in {64,128}) */
  FRT_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  FRT_ERR_CUDA = 4           /* a CUDA runtime call failed (launch, attribute query) */
} frt_status;

/*
 * frt_attn_fwd -- attention over a contiguous KV tensor (prefill, cross
 * attention and single-token decode).  The calling convention is the
 * plugin's of the "Analysis of TensorRT's low-level support for
 * FlashAttention" page (plugin sketch, enqueue): Q, K, V and O pointers, head
 * counts, query and key lengths, head dimension and the caller's stream; the
 * call returns 0 (FRT_OK) once the work is queued.  It needs no workspace.
 *
 *   q   [B, Hq,  Sq,  D] bf16      k, v  [B, Hkv, Skv, D] bf16
 *   o   [B, Hq,  Sq,  D] bf16      lse   [B, Hq, Sq] fp32, may be NULL
 *   causal: 0 or 1 (bottom-right aligned, see above); scale > 0 and finite
 *   (1/sqrt(D) in the usual model).
 *
 * Sq > 1 runs the tiled tensor-core kernel (128-query tiles, 128-key tiles,
 * fully masked key tiles skipped).  Sq == 1 runs the decode kernel in
 * cluster mode: each (sequence, KV head) is streamed by a cluster of up to
 * 16 CTAs whose partial results are merged by log-sum-exp inside the
 * cluster (distributed shared memory), in one launch and with no scratch in
 * global memory.  For a very long cache with few KV heads (fewer than about
 * 16 sequences x KV heads) frt_attn_fwd_ws spreads the keys over more of the
 * GPU.  B, Sq or Skv may be 0 (nothing to attend: o = 0, lse = -inf where
 * rows exist).
 */
FRT_API frt_status frt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Skv, int D, int causal,
                        float scale, cudaStream_t stream);

/*
 * frt_attn_fwd_ws -- frt_attn_fwd with a caller workspace, for single-token
 * decode over a long contiguous cache: Sq == 1 runs the split-KV decode of
 * frt_attn_decode_paged (any number of partitions per sequence, then the
 * log-sum-exp merge kernel), which keeps the whole GPU busy even for one
 * sequence with one KV head.  Sq > 1 is frt_attn_fwd.
 * Size query: a call with q == NULL only writes the workspace size to
 * *workspace_bytes (0 when Sq > 1) and returns FRT_OK; workspace and
 * workspace_bytes may be NULL on real calls that need none (Sq > 1).  The
 * workspace rules are those of frt_attn_decode_paged.  Sq == 1 limits B to
 * 1024.
 */
FRT_API frt_status frt_attn_fwd_ws(const void* q, const void* k, const void* v, void* o,
                                   float* lse, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                                   int causal, float scale, void* workspace,
                                   size_t* workspace_bytes, cudaStream_t stream);

/*
 * frt_attn_decode_paged -- one query token per sequence over a paged KV
 * cache ("Real-time inference optimisation" page, method paged_attention:
 * pages of 16 tokens; "FlashRT-HF-kernels" page, "Attention operators":
 * paged attention).
 *
 *   q           [B, Hq, D] bf16
 *   k_pages,
 *   v_pages     [num_pages, Hkv, page_size, D] bf16: physical pages; each
 *               (page, KV head) is one contiguous page_size x D block
 *   block_table [B, max_pages_per_seq] int32: token t of sequence b is in
 *               physical page block_table[b][t / page_size], slot
 *               t % page_size; entries past a sequence's last page are
 *               never read
 *   seq_lens    [B] int32 on the device: tokens in each sequence; a value
 *               above max_pages_per_seq * page_size is clamped to it, a
 *               negative one is read as 0
 *   o           [B, Hq, D] bf16;  lse [B, Hq] fp32, may be NULL
 *   page_size   16 in this version
 *   num_splits  number of work partitions the cache is cut into (0 = the
 *               default: enough partitions for about 18 MiB of page copies
 *               in flight, 192 on a 148-SM B200, never fewer than one or
 *               more than two per SM); every partition streams an equal
 *               share of all sequences' pages, so mixed lengths balance
 *   workspace   device scratch of *workspace_bytes bytes, 16-byte aligned.
 *               Size query: a call with q == NULL only writes the required
 *               size to *workspace_bytes and returns FRT_OK.  The size
 *               depends on B, Hq, Hkv, D and num_splits only.  Its
 *               contents need no preparation: each call writes every word
 *               it later reads, so a workspace may be reused for any call
 *               it is large enough for.  Calls that share a workspace must
 *               be ordered on the device (the same stream, or events).
 *
 * Two kernels run on `stream`: the streaming kernel, then a small merge of
 * the partitions' partial results, launched as its programmatic dependent
 * (it is scheduled early and waits on the device for the first to finish).
 * Both start by waiting for the work before them in the stream, so the call
 * is ordered like any other stream operation.
 *
 * A block-table entry outside [0, num_pages) that a sequence uses is never
 * turned into an address: the kernel checks it before issuing the copy,
 * reads that page as all zeros (keys and values 0) and sets bit 2 of the
 * device error word (frt_read_device_error).  The other sequences' results
 * are unaffected.  Tail slots of the last page of a sequence may hold
 * anything, NaN included: they never reach o.
 *
 * Size limits (FRT_ERR_UNSUPPORTED otherwise), since the kernel counts pages
 * and tokens in 32 bits: the pages of all sequences together,
 * B * max_pages_per_seq, below 2^31; a sequence's token bound,
 * max_pages_per_seq * page_size, below 2^31; and the cache's rows,
 * num_pages * Hkv * page_size, below 2^31.  Sequences may share physical
 * pages, so the first limits the block table, not the cache.
 */
FRT_API frt_status frt_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, int max_pages_per_seq,
                                 const int32_t* seq_lens, int page_size, int num_pages,
                                 void* o, float* lse, int B, int Hq, int Hkv, int D,
                                 float scale, int num_splits, void* workspace,
                                 size_t* workspace_bytes, cudaStream_t stream);

/*
 * frt_attn_prefill_paged -- chunked (or variable-length) prefill over a
 * paged KV cache: the new tokens of each sequence attend to the sequence's
 * whole cache, their own keys included ("FlashRT-HF-kernels" page,
 * "Attention operators": paged attention; the FasterTransformer read-through
 * (pptc.cn), section 3.1: context phase, requests of different lengths
 * without padding the keys).  The chunk's K/V must already be in the cache.
 *
 *   q           [B, Hq, max_q, D] bf16: sequence b's chunk in rows
 *               0..q_lens[b]-1 (the rest is padding and is not read for o)
 *   k_pages,
 *   v_pages     [num_pages, Hkv, 16, D] bf16 (as frt_attn_decode_paged)
 *   block_table [B, max_pages_per_seq] int32
 *   seq_lens    [B] int32, device: cached tokens of sequence b, its chunk
 *               included (clamped to [0, max_pages_per_seq * 16])
 *   q_lens      [B] int32, device: chunk length of sequence b (clamped to
 *               [0, max_q]); the chunk is the last q_lens[b] tokens, so with
 *               causal = 1 query i sees keys j <= i + seq_lens[b] - q_lens[b]
 *   o           [B, Hq, max_q, D] bf16; lse [B, Hq, max_q] fp32 or NULL;
 *               padding rows get o = 0, lse = -inf
 *   page_size   16
 * Runs the tiled tensor-core kernel with K/V tiles gathered page by page
 * through the block table.  Needs no workspace.  Tail slots of a sequence's
 * last page may hold anything, NaN included.  A block-table entry outside
 * [0, num_pages) is handled as in frt_attn_decode_paged: checked before any
 * copy, read as a page of zeros, reported in bit 2 of the error word.
 *
 * Size limit: max_pages_per_seq * 16 must stay below 2^31
 * (FRT_ERR_UNSUPPORTED otherwise), since a sequence's length bound is
 * computed in 32 bits.
 */
FRT_API frt_status frt_attn_prefill_paged(const void* q, const void* k_pages,
                                          const void* v_pages, const int32_t* block_table,
                                          int max_pages_per_seq, const int32_t* seq_lens,
                                          const int32_t* q_lens, int page_size, int num_pages,
                                          void* o, float* lse, int B, int Hq, int Hkv,
                                          int max_q, int D, int causal, float scale,
                                          cudaStream_t stream);

/*
 * frt_attn_decode_paged_noalloc -- frt_attn_decode_paged for callers that
 * cannot allocate device memory.  No page describes this entry point; it is
 * a convenience of this library.
 *
 * Who needs it: code whose device memory is planned once and must not call
 * cudaMalloc while it runs -- an engine plugin handed fixed buffers, a
 * real-time decode loop that cannot afford an allocation's implicit device
 * synchronisation and unbounded latency, an embedded runtime with no
 * allocator at hand.  Such a caller cannot provide frt_attn_decode_paged's
 * workspace.
 *
 * What it does: the same computation, arguments and results as
 * frt_attn_decode_paged, with the workspace taken from a fixed 16 MiB
 * buffer that the library reserves in every GPU's memory when it is loaded
 * (held until the process exits).  It allocates nothing and frees nothing.
 *   - Limit: a problem whose workspace (see frt_attn_decode_paged's size
 *     query) exceeds 16 MiB is rejected with FRT_ERR_WORKSPACE before
 *     anything runs.  At D = 128 with the default partitions that is roughly
 *     B * Hkv <= 1800 (fewer when a KV head serves more than 16 query heads).
 *   - The first call made with a given device current looks up that
 *     device's buffer address; make that first call before any stream
 *     capture on that device.
 *   - All calls on a device share the one buffer, and it keeps what the
 *     last call left in it: calls that can overlap on the device (different
 *     streams without ordering) race and corrupt each other's results.
 *     Order them, or use frt_attn_decode_paged with separate workspaces.
 */
FRT_API frt_status frt_attn_decode_paged_noalloc(const void* q, const void* k_pages,
                                                 const void* v_pages,
                                                 const int32_t* block_table,
                                                 int max_pages_per_seq, const int32_t* seq_lens,
                                                 int page_size, int num_pages, void* o,
                                                 float* lse, int B, int Hq, int Hkv, int D,
                                                 float scale, int num_splits,
                                                 cudaStream_t stream);

/*
 * frt_attn_fwd_strided -- frt_attn_fwd for tensors in any strided layout, e.g.
 * views into a fused QKV projection output [B, S, 3, H, D] or a [B, S, H, D]
 * cache, with no copy.  The Triton sketch of the "Real-time inference
 * optimisation" page (section "Flash Attention optimisation") takes a
 * stride per dimension of Q, K, V and O for the same reason.
 *   q, k, v, o  bf16; element (b, h, s, d) of a tensor is at
 *               base + b*strides[0] + h*strides[1] + s*strides[2] + d
 *               (d contiguous), with shapes [B,Hq,Sq,D], [B,Hkv,Skv,D] x2,
 *               [B,Hq,Sq,D]
 *   *_strides   host arrays of three int64 element strides (batch, head,
 *               token); each a positive multiple of 8 (the copy engine
 *               steps in 16-byte units), below 2^38
 *   lse         [B,Hq,Sq] fp32 contiguous, may be NULL
 * Every other argument as frt_attn_fwd.  All Sq (1 included) run the tiled
 * tensor-core kernel; for single-token decode over a contiguous cache
 * frt_attn_fwd (or a paged cache) is faster.  o must not overlap q, k or v,
 * and its strides must not map two elements to one address.
 */
FRT_API frt_status frt_attn_fwd_strided(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int Sq, int Skv,
                                        int D, int causal, float scale,
                                        const int64_t* q_strides, const int64_t* k_strides,
                                        const int64_t* v_strides, const int64_t* o_strides,
                                        cudaStream_t stream);

/*
 * frt_attn_decode_paged_fp8 -- frt_attn_decode_paged over an FP8 KV cache.
 * The FasterTransformer read-through (pptc.cn) keeps the KV cache quantised
 * and dequantises it before use (section 3.3, an int8 KV cache) and enables
 * FP8 on H100 and later (section 4.2).  Here the pages hold e4m3 codes
 * (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities;
 * 0x7F / 0xFF are NaN), one byte per element, in the layout of
 * frt_attn_decode_paged: [num_pages, Hkv, page_size, D] uint8.  An element
 * of KV head h stands for code * k_scale[h] (keys) or code * v_scale[h]
 * (values); every other argument means what it means for
 * frt_attn_decode_paged, and the workspace size query is the same, except
 * that num_splits = 0 means three partitions per SM when a KV head serves
 * at most 8 query heads (444 on a 148-SM B200), else two: with one byte per
 * element the kernel's arithmetic, not HBM, sets its pace.
 *   k_scale, v_scale  [Hkv] fp32 on the device, finite, 4-byte aligned
 *   D                 128 only (FRT_ERR_UNSUPPORTED otherwise)
 * The kernel converts codes to f16 (exact), multiplies q.k in f16 with fp32
 * accumulation, and rounds the softmax weights to f16 before P.V; the scales
 * are applied in fp32 to the scores and to the output.  Tail slots and pages
 * past a sequence's length may hold NaN codes: they never reach o.
 */
FRT_API frt_status frt_attn_decode_paged_fp8(const void* q, const void* k_pages,
                                             const void* v_pages, const float* k_scale,
                                             const float* v_scale, const int32_t* block_table,
                                             int max_pages_per_seq, const int32_t* seq_lens,
                                             int page_size, int num_pages, void* o, float* lse,
                                             int B, int Hq, int Hkv, int D, float scale,
                                             int num_splits, void* workspace,
                                             size_t* workspace_bytes, cudaStream_t stream);

/*
 * frt_attn_merge_lse -- combine S partial attention results of the same rows,
 * each computed over a disjoint set of keys, into the result over their
 * union.  This is the correct form of the per-page combination in the
 * "Real-time inference optimisation" page's paged_attention method (which
 * adds normalised per-page outputs): with lse = log sum_s exp(lse_s),
 *   o = sum_s exp(lse_s - lse) * o_s.
 * It is the same algebra as the online-softmax update of that page's
 * "Flash Attention optimisation" section.
 *
 *   o_parts   [S, rows, D] fp32 (rows = B * Hq), each normalised
 *   lse_parts [S, rows] fp32 natural-log LSE; -inf marks an empty part
 *   o         [rows, D] bf16;  lse [rows] fp32, may be NULL
 * A row whose parts are all empty gets o = 0, lse = -inf.  S >= 1.
 */
FRT_API frt_status frt_attn_merge_lse(const float* o_parts, const float* lse_parts, int S, int B,
                              int Hq, int D, void* o, float* lse, cudaStream_t stream);

/*
 * frt_read_device_error -- read and clear the library's device-side error
 * word on the current device (synchronises that device).  0 means no kernel
 * gave up; bit 0 = an internal wait timed out (the kernel returned without
 * finishing its outputs); bit 2 = a block-table entry outside [0, num_pages)
 * was met (that page was read as zeros, nothing outside the cache was
 * touched).  Returns FRT_ERR_CUDA if the read itself failed.
 */
FRT_API frt_status frt_read_device_error(unsigned* flags);

/*
 * frt_debug_wait_timeout -- failure-detection self-test: one thread waits on
 * an mbarrier that nothing arrives at, through the same bounded wait every
 * kernel uses.  After the wait limit (2 s) it gives up, sets bit 0 of the
 * device error word (see frt_read_device_error) and writes 2 to *returned
 * (1 would mean the wait completed, which it must not).  The context stays
 * usable.  returned: one device int32, 16-byte aligned.
 */
FRT_API frt_status frt_debug_wait_timeout(int* returned, cudaStream_t stream);

/*
 * frt_debug_fp8_decode -- diagnostic: y[i] = the value of e4m3 code codes[i]
 * as the FP8 decode kernel converts it (device arrays of n elements).  Tests
 * compare it with the e4m3 definition.  Not part of the attention path.
 */
FRT_API frt_status frt_debug_fp8_decode(const uint8_t* codes, float* y, int n,
                                        cudaStream_t stream);

/* Library version string ("major.minor.patch"). */
FRT_API const char* frt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FRT_ATTN_H_ */
