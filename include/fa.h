/*
 * fa.h: C ABI of the exact tiled attention library (sm_100a, B200).
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(Q K^T * scale) V
 * ("FlashAttention Explained: How AI Models Process Attention Faster and Use
 * Less Memory", section "Understanding Attention in Transformer Models") tile
 * by tile with an online softmax (same page, "3. Online Softmax"; "Flash
 * Attention Explained: Same Maths, Far Less Memory", "The idea: never
 * materialise the matrix"), so that the score matrix is never written to
 * device memory.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers to contiguous row-major memory
 *     owned by the caller.  bf16 tensors must be 16-byte aligned.
 *   - Layouts: q, o, dO, dq        [B, Lq, Hq, D]
 *              k, v, dk, dv        [B, Lk, Hkv, D]
 *              lse, delta          [B, Hq, Lq]     (fp32, natural log)
 *              decode q, o         [B, Hq, D];  cache [B, Lmax, Hkv, D]
 *   - D is 64 or 128; Hq must be a multiple of Hkv; query head h reads kv
 *     head h / (Hq / Hkv) (grouped-query attention, "Flash Attention
 *     Explained: Same Maths, Far Less Memory", "What it does not solve").
 *   - causal != 0 allows key j for query i when j <= i + (Lk - Lq)
 *     (bottom-right alignment).  A query with no allowed key gets O = 0 and
 *     LSE = -inf.
 *   - scale must be finite and > 0 (1/sqrt(D) is the pages' choice).
 *   - stream is a cudaStream_t (may be 0).  Every call only enqueues work: it
 *     never synchronises and never allocates.  Arguments are checked before
 *     anything is launched; a bad argument returns FA_ERR_INVALID_ARG or
 *     FA_ERR_UNSUPPORTED and launches nothing.  A failed launch returns
 *     FA_ERR_CUDA.  Device-side faults surface at the caller's next
 *     synchronisation; a kernel wait that runs out of time is reported by
 *     fa_device_status() (the kernel then returns instead of hanging).
 *   - The library keeps two device words of state (the device status) and a
 *     per-device record of kernel attributes set; calls are thread-safe.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* same type as cudaStream_t */

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, workspace too small */
  FA_ERR_UNSUPPORTED = 2, /* valid but not implemented here (e.g. D not in {64,128}) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, tensor map) */
  FA_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (see fa_device_status) */
  FA_ERR_DEVICE_INDEX = 5 /* debug build: a kernel's store index check failed (see fa_device_status) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP32 = 1 } fa_dtype;

/* Version of this ABI (incremented on any signature change). */
int fa_abi_version(void);

/* Static text for a status code; never NULL. */
const char* fa_status_string(int status);

/*
 * 1 for the debug build (compiled with FA_DEBUG: every global store of every
 * kernel checks its index against the size of its tensor; an out-of-range
 * store is skipped and fa_device_status() reports FA_ERR_DEVICE_INDEX), else
 * 0.  The debug build is libfa46_debug.so beside libfa46.so; no counterpart
 * on the pages.
 */
int fa_debug_build(void);

/*
 * Prefill forward.  Reads q, k, v (bf16); writes o (bf16) and, when lse is
 * not NULL, lse (fp32, ln of the softmax denominator including the max).
 * Lq == 0 is a no-op; Lk == 0 writes O = 0 and LSE = -inf.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int causal,
                 fa_stream_t stream);

/* As fa_fwd, with the output dtype of o chosen (FA_BF16 or FA_FP32). */
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int causal,
                    int o_dtype, fa_stream_t stream);

/*
 * Prefill forward on e4m3 (FP8) inputs ("FlashAttention Explained ...",
 * section "FlashAttention-4 and Newer Research": later versions rework
 * precision among other things).  q, k, v hold one e4m3 byte per element in
 * the usual layouts; the value of an element is its e4m3 value times the
 * tensor's scale (q_scale, k_scale, v_scale: finite, > 0).  Both products run
 * on the tensor cores in e4m3 with fp32 accumulation: S = (q k^T) * q_scale *
 * k_scale * scale, and P (kept in e4m3, scaled by 2^8 against the running
 * max) times v.  o (o_dtype) and lse are as in fa_fwd, in the dequantized
 * units.  The only rounding beyond fa_fwd's is that of P to e4m3 (relative
 * 2^-4, or 2^-18 of the row's largest probability absolute), which moves O by
 * at most that much of the spread of the attended v rows; the LSE uses the
 * unrounded probabilities.  D must be 128 (else FA_ERR_UNSUPPORTED).
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale,
                     float v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Lq, int Lk,
                     int D, float scale, int causal, int o_dtype, fa_stream_t stream);

/*
 * Backward ("FlashAttention Explained ...", section "More Efficient
 * Backpropagation"; "How FlashAttention Speeds Up LLM Attention", "Recompute
 * probabilities for training"): probabilities are recomputed per tile from q,
 * k and the saved lse instead of being stored.  Reads q, k, v, o, dO (bf16)
 * and lse (fp32, as written by fa_fwd); writes dq [B,Lq,Hq,D], dk and dv
 * [B,Lk,Hkv,D] in grad_dtype (FA_BF16 or FA_FP32).  dk/dv of a kv head are the
 * sums over its Hq/Hkv query heads.  The products run on fp16 operands: each
 * input tensor is scaled by a power of two (chosen on the device from its
 * largest magnitude) so that its bf16 values convert to fp16 exactly, P and
 * dS enter the products as fp16, and the scales are taken out of the results
 * exactly; an input holding inf or NaN gives non-finite gradients.  workspace
 * is caller-owned device memory of at least fa_bwd_workspace_size() bytes
 * (256-byte aligned: the fp32 dQ accumulator, the LSE and Delta rows, the
 * scaled fp16 copies of q and dO, the input maxima and the main kernel's work
 * counter); its contents on entry do not matter.  Calls that share one
 * workspace must be ordered on one stream.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Lq, int D);
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int causal,
                 int grad_dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Split-KV decode ("Flash Attention Explained: Same Maths, Far Less Memory",
 * "Where you actually feel it"): one query per (sequence, head) against the
 * first seqlens[b] rows of a contiguous cache.  q [B,Hq,D] bf16; k_cache,
 * v_cache [B,Lmax,Hkv,D] bf16; seqlens int32 [B] on the device (values are
 * clamped to [0, Lmax]; rows at or past seqlens[b] are never read into the
 * result); o [B,Hq,D] in o_dtype; lse [B,Hq] fp32 or NULL.  The cache is cut
 * into chunks of fa_decode_chunk() keys; each chunk's partial result goes to
 * the workspace (>= fa_decode_workspace_size() bytes, 256-byte aligned) and a
 * second kernel combines them.  Two launches on `stream`.
 */
int fa_decode_chunk(void);
size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int D);
fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                            const int* seqlens, void* o, float* lse,
                            int B, int Hq, int Hkv, int Lmax, int D, float scale,
                            int o_dtype, void* workspace, size_t workspace_bytes,
                            fa_stream_t stream);

/*
 * Decode with the new token's K/V appended to the cache in the same call
 * ("FlashAttention Explained ...", section "FlashAttention vs. KV Cache": the
 * cache keeps the past keys and values and each generated token adds its
 * own).  k_new, v_new [B,Hkv,D] bf16 are the new token's rows.  For every
 * sequence b with seqlens[b] < Lmax, the query attends over the seqlens[b]
 * cached rows plus the new row (seqlens[b] + 1 keys), and the new rows are
 * written into k_cache / v_cache at row seqlens[b] (no other cache row is
 * touched).  seqlens is NOT advanced: the caller adds 1 after the call.  A
 * sequence with seqlens[b] >= Lmax has no room: nothing is attended or written
 * for it (o = 0, lse = -inf) and fa_device_status() reports
 * FA_ERR_INVALID_ARG.  Workspace: at least fa_decode_workspace_size(B, Hq,
 * Lmax + 1, D) bytes.  Otherwise as fa_decode_splitkv.
 */
fa_status fa_decode_append_splitkv(const void* q, const void* k_new, const void* v_new,
                                   void* k_cache, void* v_cache, const int* seqlens, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                   int o_dtype, void* workspace, size_t workspace_bytes,
                                   fa_stream_t stream);

/*
 * Decode from a paged KV cache ("Flash Attention Explained: Speed From Memory
 * Movement", section "What changed in 2026": decode-phase variants, and its
 * linked note "Paged Attention: Fixing the KV Cache Memory Problem").  The
 * rows live in a pool of fixed-size pages, k_pages / v_pages
 * [num_pages, page_size, Hkv, D] bf16; page_table [B, pages_per_seq] int32 on
 * the device gives, for sequence b, the pool index of its p-th page, so that
 * cache row r of sequence b is row r % page_size of page
 * page_table[b][r / page_size].  page_size must be a multiple of 16.  Only
 * the table entries that cover rows below seqlens[b] (and, with append, row
 * seqlens[b]) are read; an entry outside [0, num_pages) is never dereferenced:
 * its rows are skipped and fa_device_status() reports FA_ERR_INVALID_ARG.
 * k_new / v_new: NULL for plain decode over seqlens[b] rows (clamped to
 * pages_per_seq * page_size); or the new token's rows [B,Hkv,D], attended as
 * key seqlens[b] and written at that row, as in fa_decode_append_splitkv (the
 * page holding that row must already be in the table).  Workspace: at least
 * fa_decode_workspace_size(B, Hq, pages_per_seq * page_size + (append ? 1 : 0),
 * D) bytes.  Otherwise as fa_decode_splitkv.
 */
fa_status fa_decode_paged_splitkv(const void* q, const void* k_new, const void* v_new,
                                  void* k_pages, void* v_pages, const int* page_table,
                                  const int* seqlens, void* o, float* lse,
                                  int B, int Hq, int Hkv, int num_pages, int page_size,
                                  int pages_per_seq, int D, float scale, int o_dtype,
                                  void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Split-KV decode that allocates nothing and takes no workspace.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot
 * obtain device memory at the moment they run a decode step: for example an
 * engine plugin or serving loop whose memory is fixed when it starts and that
 * may not call cudaMalloc later (cudaMalloc can block and synchronise the
 * device, which a per-token latency budget cannot absorb), or a foreign-
 * language caller that can only hand over the tensors it already owns.
 *
 * Arguments, layouts and results are those of fa_decode_splitkv without the
 * workspace pair; the caller still owns and passes every input and output.
 * The partial results live instead in one file-scope device array of
 * FA_DECODE_STATIC_SCRATCH_BYTES bytes inside the library.  Every GPU that
 * loads the library holds that array until the process exits.  A
 * configuration whose fa_decode_workspace_size() exceeds it returns
 * FA_ERR_UNSUPPORTED and launches nothing.
 *
 * The first call on a device looks up the array's address on that device
 * (with that device current).  Under CUDA's lazy module loading that first
 * look-up may also be what loads the library's kernels onto the device and
 * reserves the array there, which can take time and synchronise; so make one
 * warm-up call of this entry point on every device at start-up (before any
 * stream capture and before the latency-critical loop).
 * All calls share the one array and it keeps the last call's contents; nothing
 * in it has to start at zero, because every partial result the combine step
 * reads is written earlier in the same call.  Calls whose kernels may overlap
 * on the GPU (different streams, or threads without ordering between them)
 * race on the array and corrupt each other's results: order such calls.
 * Never calls cudaMalloc, cudaFree or any allocating library routine.
 */
#define FA_DECODE_STATIC_SCRATCH_BYTES (40u * 1024u * 1024u)
fa_status fa_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache,
                                   const int* seqlens, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                   int o_dtype, fa_stream_t stream);

/*
 * Combine partial results over disjoint key sets (the merge step of split-KV
 * decode; "How FlashAttention Speeds Up LLM Attention": partial results kept
 * on the same numerical scale).  o_part [B,Hq,max_splits,D] fp32 holds
 * normalised partial outputs, lse_part [B,Hq,max_splits] fp32 their natural
 * log-sum-exps (-inf for an empty part).  num_splits [B] int32 on the device
 * gives how many leading parts of sequence b are valid (NULL: all
 * max_splits).  Writes o [B,Hq,D] in o_dtype and lse [B,Hq] (or NULL):
 * lse = ln sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s.
 */
fa_status fa_decode_combine(const float* o_part, const float* lse_part, const int* num_splits,
                            void* o, float* lse, int B, int Hq, int D, int max_splits,
                            int o_dtype, fa_stream_t stream);

/*
 * Merge of two attention results over disjoint key sets, in the prefill
 * layout: the step that joins the partial results of context-parallel (ring)
 * prefill, where a rank's queries meet the key/value blocks one at a time
 * ("How FlashAttention Speeds Up LLM Attention": partial results kept on a
 * common numerical scale are combined; "FlashAttention Explained ...",
 * "Longer Context Windows").  o_a, o_b [B,L,H,D] fp32 are normalised outputs
 * over the two key sets, lse_a, lse_b [B,H,L] fp32 their natural
 * log-sum-exps (-inf for a row with no key in that set).  Writes
 *   lse_out = ln(e^lse_a + e^lse_b),  o_out = e^(lse_a - lse_out) o_a + e^(lse_b - lse_out) o_b
 * (o_out in o_dtype; a row empty on both sides gets 0 and -inf).  o_out may
 * be o_a or o_b (fp32) and lse_out lse_a or lse_b (in-place accumulation);
 * lse_out may be NULL.  D must be a multiple of 4.
 */
fa_status fa_attn_merge(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b,
                        void* o_out, float* lse_out, int B, int H, int L, int D, int o_dtype,
                        fa_stream_t stream);

/*
 * Device status of the current device: *code receives 0 (ok), FA_ERR_TIMEOUT
 * when some kernel's bounded wait ran out since the last reset, or
 * FA_ERR_INVALID_ARG when a kernel met device-side input it could not honour
 * (a page index outside the pool, a sequence without room for an appended
 * row) and skipped that work, or FA_ERR_DEVICE_INDEX when, in the debug
 * build, a store failed its index check; *where a code naming the place (first
 * event since the reset wins).  Synchronises `stream`.  reset != 0 clears the status.
 */
fa_status fa_device_status(int* code, int* where, int reset, fa_stream_t stream);

/*
 * Upper bound, in nanoseconds, on any single wait inside a kernel (default
 * 2e9).  Process-wide; affects launches made after the call.
 */
void fa_set_wait_limit_ns(unsigned long long ns);

/*
 * Self-test of the bounded wait: launches one block that waits on a barrier
 * nothing ever completes, with a limit of wait_ns nanoseconds; the kernel
 * records FA_ERR_TIMEOUT in the device status and returns.
 */
fa_status fa_selftest_wait_timeout(unsigned long long wait_ns, fa_stream_t stream);

/*
 * Register guard of the tensor-core kernels (for tests).  The forward and
 * backward kernels hand registers between their warpgroups (setmaxnreg), which
 * is only safe when a thread is launched with exactly the registers the split
 * assumes; before the first launch of each kernel instantiation the library
 * compares the compiled register count with that figure and refuses the launch
 * (FA_ERR_UNSUPPORTED) on a mismatch.  For the instantiation (bwd, D, causal)
 * this reports, when the pointers are not NULL: *state, that instantiation's
 * cached check result (0 not yet checked, 1 match, 2 mismatch; never changed by
 * this call); *expected_regs, the figure the split assumes; *num_regs, the
 * compiled count (queried from the runtime, which needs a GPU; pass NULL to
 * skip).  D must be 64 or 128, or -128 for the e4m3 forward (bwd = 0).  No
 * counterpart on the pages.
 */
fa_status fa_launch_guard(int bwd, int D, int causal, int* num_regs, int* expected_regs, int* state);

/*
 * Self-test of the FMA-pipe exponential the forward kernel can use for part of
 * its probabilities (off in this build: every share measured slower than the
 * MUFU unit alone): y[i] = 2^x[i] for n device floats, computed exactly as that
 * path does (round-to-nearest split, fitted cubic, exponent add; inputs below
 * -126 give a tiny positive value).  For tests only.
 */
fa_status fa_selftest_exp2_poly(const float* x, float* y, int n, fa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */
