/*
 * gqa_attn: forward scaled-dot-product attention with grouped-query heads on
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 *     O   = softmax(scale * Q K^T + causal mask) V
 *     LSE = log(sum_t exp(scale * q . k_t))      (natural log, visible keys only)
 *
 * Query head h reads K/V head h / (Hq / Hkv): contiguous groups of Hq/Hkv query
 * heads share one K/V head ("ggml-org/llama.cpp PR #28507", Setup: GQA 8, and
 * the FLASH_ATTN_EXT case list: nr23 broadcast ratio).
 *
 * Causal mask: key t is visible to query row s iff t <= q_offset + s, i.e. the
 * Sq new queries sit at positions q_offset .. q_offset+Sq-1 of the key
 * sequence (prefill at depth, speculative-verify rows).  q_offset >= 0, so
 * every row sees at least key 0.
 *
 * Layouts (contiguous, row-major, element counts):
 *     q, out        [B, Sq,  Hq,  D]
 *     k, v          [B, Skv, Hkv, D]       bf16
 *     lse           [B, Hq,  Sq]           fp32
 *     partial_out   [S, B, Sq, Hq, D]      fp32 (S = num_splits)
 *     partial_lse   [S, B, Hq, Sq]         fp32
 * q, k, v are bf16.  out is bf16 or fp32 (out_dtype).
 *
 * Ownership: every buffer is allocated and owned by the caller and is DEVICE
 * memory of the current CUDA device; the library allocates nothing per call.
 * It keeps only one device status word per device (for attn_last_status).
 *
 * Asynchrony: every compute call is enqueued on `stream` (a cudaStream_t
 * passed as void*; NULL means the legacy default stream) and returns at once.
 * The return value covers argument checks and the launch itself.  A kernel
 * that gives up on a stalled pipeline (a bounded wait that ran out) records
 * ATTN_ERR_TIMEOUT in the device status word; attn_last_status() reads it.
 *
 * Errors: argument errors are detected on the host before any CUDA call and
 * leave every output untouched.
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, Hq % Hkv != 0, bad split count */
  ATTN_ERR_UNSUPPORTED = -2,  /* a head dim or row count this build has no kernel for */
  ATTN_ERR_ALIGNMENT = -3,    /* q/k/v/out/partials not 16-byte aligned, lse not 4-byte aligned */
  ATTN_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed (no device, launch error) */
  ATTN_ERR_TIMEOUT = -5,      /* a kernel's bounded pipeline wait ran out (device status) */
  ATTN_ERR_TOO_LARGE = -6     /* attn_decode_noalloc: partials exceed the fixed scratch array */
} attn_status;

typedef enum { ATTN_BF16 = 0, ATTN_F32 = 1, ATTN_FP8_E4M3 = 2 } attn_dtype;

/*
 * Prefill: all Sq query rows against all Skv keys in one pass.  The flash
 * formulation with an online softmax keeps a running per-row (max, rowsum) and
 * rescales the output accumulator ("Anbeeld/beellama.cpp PR #149", Overview:
 * warp-shuffle reduction and fp32 rescale; every tile publishes its (max,
 * rowsum)); K/V tiles are staged in shared memory and reused by all query rows
 * of a tile ("ggml-org/llama.cpp PR #28507", the staging change;
 * "AstrAI commit log, gqa_prefill_attn_mma.cuh", cp.async K/V loads and the
 * pre-scaled Q, whose scale this library applies in fp32 instead of rounding
 * Q*scale to bf16).
 *
 *   D          64, 128, 256 or 512 (else ATTN_ERR_UNSUPPORTED).  D = 512 runs the
 *              split-KV kernel with one split and the query rows cut into
 *              chunks of 80 / (Hq/Hkv) positions per CTA, writing O and LSE
 *              directly; it needs Hq/Hkv <= 32 (else ATTN_ERR_UNSUPPORTED)
 *   scale      > 0 and finite (else ATTN_ERR_INVALID_ARG)
 *   causal     0 or 1; q_offset >= 0
 *   out_dtype  ATTN_BF16 or ATTN_F32 (round to nearest even for bf16)
 *   lse        may be NULL (then no LSE is written)
 */
int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal,
                 float scale, int out_dtype, void* stream);

/*
 * Split-KV decode ("flash decoding"): the keys are cut into num_splits
 * contiguous chunks of c = ceil(Skv / num_splits) keys; split s covers keys
 * [s*c, min((s+1)*c, Skv)).  Each split writes its own normalised partial
 * output and its log-sum-exp.  EVERY split publishes, including a split that
 * holds no key or whose keys are all masked for a row: that row gets
 * partial_lse = -inf and partial_out = 0 ("Anbeeld/beellama.cpp PR #149",
 * Overview, the ub>64 fix: whole-tile blocks must publish their (max, rowsum)
 * or the merge silently drops their rows).
 *
 *   D            64, 128, 256 or 512 (else ATTN_ERR_UNSUPPORTED); the pages'
 *                kernels carry D = 64 K/V heads ("Anbeeld/beellama.cpp PR
 *                #149", Base: v0.4.7, D=64 KV-head support; the HEAD_DIM
 *                dispatch of "ViperEkura/AstrAI commit 7ba43a7,
 *                gqa_prefill_attn_mma.cuh")
 *   rows         R = (Hq/Hkv) * Sq query rows share one K/V head; R rounded up
 *                to a multiple of 16 must satisfy (2 + ceil(D/128)) * R16 <= 256
 *                (else ATTN_ERR_UNSUPPORTED): at most 80 rows for D = 64 and
 *                D = 128, 64 for D = 256, 32 for D = 512
 *   num_splits   1 <= num_splits <= Skv (else ATTN_ERR_INVALID_ARG)
 *   partial_out  num_splits*B*Sq*Hq*D floats; partial_lse num_splits*B*Hq*Sq
 */
int attn_decode_split(const void* q, const void* k, const void* v, float* partial_out,
                      float* partial_lse, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                      int q_offset, int causal, float scale, int num_splits, void* stream);

/*
 * Merge of split partials by their log-sum-exp ("Anbeeld/beellama.cpp PR
 * #149", review note on the combine kernel for parallel_blocks > 1):
 *     M = max_s lse_s;  w_s = exp(lse_s - M);
 *     out = sum_s w_s * O_s / sum_s w_s;   lse = M + log(sum_s w_s).
 * Splits with lse = -inf get weight 0.  lse may be NULL.
 *   D            any multiple of 4 in [4, 1024] (else ATTN_ERR_UNSUPPORTED)
 * The merge is launched with programmatic stream serialization: it may be
 * scheduled before the kernel ahead of it on the stream has finished (the
 * split-KV kernel allows that from its start), and every block waits for
 * that kernel to complete, with its writes visible, before it reads
 * anything; stream order is kept.
 */
int attn_merge(const float* partial_out, const float* partial_lse, void* out, float* lse,
               int B, int Hq, int Sq, int D, int num_splits, int out_dtype, void* stream);

/* Bytes of partial_out plus partial_lse that attn_decode_split needs; 0 on
 * invalid sizes.  Both pieces start 16-byte aligned if the caller places
 * partial_lse at partial_out + num_splits*B*Sq*Hq*D floats. */
size_t attn_decode_workspace_bytes(int B, int Hq, int Sq, int D, int num_splits);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: ATTN_OK; ATTN_ERR_TIMEOUT if a kernel gave up on a
 * stalled pipeline since the last call; ATTN_ERR_INVALID_ARG if a device-side
 * sequence length (attn_kv_view.seq_lens) was outside [0, Skv] and was
 * clamped.  ATTN_ERR_CUDA if the sync fails. */
int attn_last_status(void* stream);

/* Human-readable name of a status code (static storage). */
const char* attn_status_string(int status);

/*
 * Self-test of the bounded wait: launches one CTA that waits on an mbarrier
 * nothing will ever complete, with the given limit in nanoseconds (clamped to
 * [1e3, 5e9]).  The wait gives up, the kernel records ATTN_ERR_TIMEOUT and
 * exits normally; read it back with attn_last_status().  No hang, no fault.
 */
int attn_watchdog_selftest(unsigned long long limit_ns, void* stream);

/*
 * Allocation-free split-KV decode + merge.  The pages have no counterpart:
 * this serves callers that cannot allocate a device workspace (a plugin host
 * that owns the whole device memory pool and hands an operator only its
 * inputs and outputs; a latency-critical decode loop that must not call
 * cudaMalloc, which can synchronise the device).
 *
 * Same arguments and results as attn_decode_split followed by attn_merge into
 * out [B,Sq,Hq,D] (out_dtype) and lse [B,Hq,Sq] (may be NULL), but the split
 * partials live in one fixed device array inside the library, of
 * ATTN_NOALLOC_SCRATCH_BYTES bytes, held by every device that loads the
 * library until the process exits.  The library calls no cudaMalloc, cudaFree
 * or other allocating routine.
 *   - Capacity: num_splits*B*Sq*Hq*D*4 bytes (rounded up to 256) plus
 *     num_splits*B*Hq*Sq*4 bytes must fit, else ATTN_ERR_TOO_LARGE (checked on
 *     the host before anything is launched).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; nothing
 *     in it needs clearing, since each call's split kernel writes every
 *     partial that its merge reads.  Calls whose kernels overlap on the GPU
 *     (different streams or host threads) race on it: serialise them.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)
int attn_decode_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal,
                        float scale, int num_splits, int out_dtype, void* stream);

/*
 * Optional terms of the attention logit, from the parameters of the
 * FLASH_ATTN_EXT operator ("ggml-org/llama.cpp PR #28507", Crash 1: the test
 * case list carries sinks, max_bias and logit_softcap).  With z the scaled
 * logit scale * q.k_t of query row s (position pos = q_offset + s) and key t:
 *
 *   softcap > 0          z = softcap * tanh(z / softcap)
 *   alibi_max_bias > 0   z = z + slope_h * (t - pos), slope_h geometric per
 *                        head: n2 = largest power of two <= Hq,
 *                        m0 = 2^(-max_bias / n2), m1 = 2^(-max_bias / (2 n2)),
 *                        slope_h = m0^(h+1) for h < n2, else m1^(2(h-n2)+1)
 *   sinks != NULL        device array [Hq] of fp32 sink logits: exp(sinks[h])
 *                        joins the softmax denominator (and the LSE), with no
 *                        value row
 *   window > 0           key t is visible only if pos - window < t; needs
 *                        causal = 1 and q_offset + Sq <= Skv (every query
 *                        position has its key), else ATTN_ERR_UNSUPPORTED
 *   mask != NULL         additive bf16 mask (the `mask` parameter of the same
 *                        test case): z += mask[b*mask_stride_seq +
 *                        s*mask_stride_row + t] for t < Skv, after softcap and
 *                        ALiBi; -inf removes the key.  mask_stride_seq = 0
 *                        shares one [Sq, Skv] mask across the batch.  A row
 *                        whose every visible key is masked gets O = 0 and
 *                        LSE = -inf (or the sink logit with a sink).
 *
 * Zero / NULL fields are off.  softcap and alibi_max_bias must be finite and
 * >= 0, window >= 0 (else ATTN_ERR_INVALID_ARG); sinks must be 4-byte aligned
 * (else ATTN_ERR_ALIGNMENT); the mask must be 2-byte aligned (else
 * ATTN_ERR_ALIGNMENT) with non-negative strides (else ATTN_ERR_INVALID_ARG);
 * rows that start 16-byte aligned (mask 16-byte aligned, strides multiples of
 * 8) are read with vector loads, others one element at a time.
 * The caller owns *opt, the sink array and the mask; the call reads *opt on
 * the host before it returns and the arrays on the device, in stream order.
 */
typedef struct attn_options {
  float softcap;
  float alibi_max_bias;
  const float* sinks;
  int window;
  const void* mask;             /* bf16, or NULL */
  long long mask_stride_seq;    /* elements between sequences (0: shared) */
  long long mask_stride_row;    /* elements between query rows */
} attn_options;

/* attn_prefill with the optional terms of *opt (opt may be NULL). */
int attn_prefill_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                    int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal,
                    float scale, int out_dtype, const attn_options* opt, void* stream);

/* attn_decode_split with softcap, ALiBi and window from *opt (opt may be
 * NULL).  Sinks belong to the merge, which adds them once per row:
 * opt->sinks must be NULL here (else ATTN_ERR_INVALID_ARG). */
int attn_decode_split_ex(const void* q, const void* k, const void* v, float* partial_out,
                         float* partial_lse, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                         int q_offset, int causal, float scale, int num_splits,
                         const attn_options* opt, void* stream);

/* attn_merge with optional sink logits (device [Hq] fp32, may be NULL):
 * M = max(max_s lse_s, sink_h), denominator sum_s w_s + exp(sink_h - M). */
int attn_merge_ex(const float* partial_out, const float* partial_lse, void* out, float* lse,
                  int B, int Hq, int Sq, int D, int num_splits, int out_dtype, const float* sinks,
                  void* stream);

/*
 * A K/V cache view for decode: strided, optionally paged, optionally with a
 * length per sequence (paged K/V as in the paged indexer of the
 * "amd-sriram/vllm PR #32" Validation section; strided K/V views as in the
 * kv_view and permute parameters of the FLASH_ATTN_EXT test cases in
 * "ggml-org/llama.cpp PR #28507", Crash 1).  All strides are in elements,
 * D is innermost and contiguous.
 *
 * Unpaged (block_table == NULL): key t of sequence b, K/V head kvh is at
 *   k + b*stride_seq + t*stride_token + kvh*stride_head   (same for v)
 * for t < Skv.
 * Paged: logical page j of sequence b is physical page block_table[b*max_pages + j];
 * key t of sequence b is row t % page_size of page block_table[b*max_pages + t / page_size]:
 *   k + page*stride_seq + (t % page_size)*stride_token + kvh*stride_head
 * with 0 <= page < num_pages.  page_size is 16, 32, 64 or a multiple of 128;
 * Skv must equal max_pages * page_size.  A physical page index outside
 * [0, num_pages) reads as zeros (never out of bounds).
 *
 * seq_lens (device [B] int32, or NULL): sequence b has min(seq_lens[b], Skv)
 * keys and its Sq query rows sit at positions len_b - Sq + s (q_offset is
 * ignored); rows at a negative position see no key.  A negative or too large
 * length is clamped to [0, Skv] and sets ATTN_ERR_INVALID_ARG in the device
 * status word (see attn_last_status).  Without seq_lens every sequence has Skv
 * keys and q_offset applies.
 *
 * Quantised K/V (kv_dtype = ATTN_FP8_E4M3): k and v hold one e4m3 code per
 * element and K = e4m3(code) * k_scale[kvh], V = e4m3(code) * v_scale[kvh]
 * (the quantised K/V cache of "ggml-org/llama.cpp PR #28507", Setup, and
 * "Anbeeld/beellama.cpp PR #149", Overview).  The tensor cores read the codes
 * directly (kind::f8f6f4); Q and P enter as two e4m3 planes each (hi + lo),
 * which carry a bf16 value's 8 significant bits.  Q is scaled by a power of
 * two per CTA first, so it needs no range condition.  k_scale and v_scale
 * must be finite and > 0 (not checked on the device).
 *
 * Alignment: k, v 16-byte aligned; stride_seq, stride_token and stride_head
 * multiples of 16 bytes (8 bf16 or 16 fp8 elements) and each below 2^37
 * elements, else ATTN_ERR_ALIGNMENT / ATTN_ERR_INVALID_ARG; k_scale and
 * v_scale non-NULL and 4-byte aligned for fp8 (else ATTN_ERR_INVALID_ARG).
 * The caller owns every buffer.
 *
 * Head sizes (head_dim_v): K has D columns per head (D = the Q head size
 * argument), V has Dv = head_dim_v columns (0 means Dv = D), and O and the
 * partials have Dv columns: out and partial_out are [.., Hq, Dv] instead of
 * [.., Hq, D].  Pairs with Dv != D are (D, Dv) = (576, 512), (320, 256) and
 * (192, 128), bf16 only ("ggml-org/llama.cpp PR #28507", the FLASH_ATTN_EXT
 * cases with hsk=320, hsv=256 and the v_is_view_of_k flag; "Anbeeld/beellama.cpp
 * PR #149", the D256 tile follow-up and the (576, 512) rows of the review).
 * V may be a view of K: v = k with the same strides reads the first Dv
 * columns of each K row (multi-head latent attention caches).  Other pairs
 * give ATTN_ERR_UNSUPPORTED.
 *
 * V strides (v_stride_*): V's elements sit at v + (same index expression)
 * with v_stride_seq, v_stride_token and v_stride_head in place of K's, for
 * separate K and V tensors of different widths or layouts.  All three 0
 * means V shares K's strides; otherwise each obeys the rules for K's.
 */
typedef struct attn_kv_view {
  const void* k;            /* bf16 */
  const void* v;            /* bf16 */
  long long stride_seq;     /* between sequences (unpaged) or pages (paged) */
  long long stride_token;   /* between consecutive keys */
  long long stride_head;    /* between K/V heads */
  const int* block_table;   /* device [B, max_pages], or NULL: unpaged */
  int max_pages;            /* columns of block_table */
  int page_size;            /* keys per page */
  int num_pages;            /* physical pages in the cache */
  const int* seq_lens;      /* device [B], or NULL */
  int kv_dtype;             /* ATTN_BF16 or ATTN_FP8_E4M3 */
  const float* k_scale;     /* fp8: device [Hkv], K = code * k_scale[kvh] */
  const float* v_scale;     /* fp8: device [Hkv], V = code * v_scale[kvh] */
  int head_dim_v;           /* V and O head size Dv, or 0: Dv = D */
  long long v_stride_seq;   /* V's own strides, or all three 0: V uses K's */
  long long v_stride_token;
  long long v_stride_head;
} attn_kv_view;

/*
 * attn_decode_split over a K/V view (optional logit terms in *opt, which may
 * be NULL; sinks belong to attn_merge_ex).  Splits: chunk = ceil(len_b /
 * num_splits) keys of sequence b per split, rounded up to a multiple of 128
 * when paged so that no 128-key tile crosses a page; splits past the end
 * publish lse = -inf and O = 0.  With head_dim_v = Dv != D the partials are
 * [S, B, Sq, Hq, Dv] and the row limit reads (2 + ceil(Dv/128)) * R16 <= 256; merge
 * them with attn_merge at D = Dv.  Other arguments, limits and errors as in
 * attn_decode_split.
 */
int attn_decode_split_kv(const void* q, const attn_kv_view* kv, float* partial_out, float* partial_lse,
                         int B, int Hq, int Hkv, int Sq, int Skv, int D, int q_offset, int causal,
                         float scale, int num_splits, const attn_options* opt, void* stream);

/*
 * Split-KV decode and merge in ONE launch ("flash decoding" with the combine
 * fused into the split kernel): the key ranges of one (sequence, K/V head)
 * run as one thread-block cluster of n CTAs; each CTA leaves its (max,
 * rowsum) and unnormalised O in its shared memory and every CTA merges a
 * slice of the output columns from all n over distributed shared memory
 * (the last-CTA combine of "Anbeeld/beellama.cpp PR #149", review of the
 * combine kernel for parallel_blocks > 1, done by all CTAs at once).  No
 * partial goes to HBM, no workspace is needed.
 *   n            the largest power of two <= min(num_splits, 8): key range
 *                k of n covers keys [k c, (k+1) c), c = ceil(len / n)
 *                (rounded up to 128 when paged); the result is the attention
 *                of attn_decode_split_kv + attn_merge_ex with n splits.
 *                When to call it: it saves the merge launch and the partials'
 *                round trip through HBM, but it runs only B * Hkv * n CTAs
 *                (n <= 8), where attn_decode_split_kv runs B * Hkv * num_splits
 *                (grouped to fill the GPU).  Measured on B200 (148 SMs, two
 *                CTAs each): with B * Hkv * n >= 2 * 148 it is faster (8-row
 *                verify, B4 Hkv8 D128: 98 vs 111 us per step); with fewer
 *                CTAs it is not (B16 Hkv1 D512: 118 vs 111 us), so such
 *                shapes should call attn_decode_split_kv + attn_merge_ex
 *   out, lse     as attn_merge_ex's: out [B, Sq, Hq, Dv] (out_dtype), lse
 *                [B, Hq, Sq] fp32 or NULL; opt->sinks apply here
 *   limits       those of attn_decode_split_kv, and the merge's shared memory
 *                (RP x Dv fp32 plus 17 RP floats) must fit the K/V ring the
 *                launch gets, else ATTN_ERR_UNSUPPORTED
 */
int attn_decode_fused(const void* q, const attn_kv_view* kv, void* out, float* lse, int B, int Hq, int Hkv,
                      int Sq, int Skv, int D, int q_offset, int causal, float scale, int num_splits,
                      int out_dtype, const attn_options* opt, void* stream);

/*
 * Prefill over a K/V view: attn_prefill_ex with K and V described by *kv
 * (strides, paging, lengths per sequence, fp8 codes, Dv != D).  out is
 * [B, Sq, Hq, Dv].  With seq_lens, q_offset is ignored and the Sq rows of
 * sequence b sit at positions len_b - Sq + s, as in attn_decode_split_kv.
 *   - D = Dv in {64, 128, 256}, or D = 192 with Dv = 128; bf16, unpaged, no
 *     seq_lens: the prefill kernel, reading K and V through the view's
 *     strides.
 *   - otherwise (D = Dv = 512, the pairs with Dv != D, paged, fp8 or
 *     seq_lens): the split-KV kernel with one split and the query rows cut
 *     into chunks per CTA, writing O and LSE directly, as attn_prefill does
 *     at D = 512.  Dims: D = Dv in {64 (bf16 only), 128, 256, 512}, or a pair listed under
 *     attn_kv_view; Hq/Hkv <= 32.  Else ATTN_ERR_UNSUPPORTED.
 * Arguments, options (*opt may be NULL; sinks apply here), alignment and
 * errors otherwise as in attn_prefill_ex and attn_decode_split_kv.
 */
int attn_prefill_kv(const void* q, const attn_kv_view* kv, void* out, float* lse, int B, int Hq, int Hkv,
                    int Sq, int Skv, int D, int q_offset, int causal, float scale, int out_dtype,
                    const attn_options* opt, void* stream);

/* Library version, e.g. 0x000500 for 0.5.0. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
