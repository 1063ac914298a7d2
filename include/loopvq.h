/*
 * loopvq.h -- C ABI of libloopvq, the B200 (sm_100a) hot path of LoopVQ:
 * loop-axis vector-quantized KV-cache encode and decode attention for
 * looped transformers.
 *
 * Method (LoopVQ project page, mscheong01.github.io/loopvq):
 *   - "Method", figure "Overview of LoopVQ" and "Component 1 -- Loop-axis
 *     vector quantization": one codebook index covers G/Tc channels of each
 *     of Tc consecutive loop steps; at inference each loop step reads the
 *     shared index through its own slice of the codebook.
 *   - "Serving in SGLang": a new token's keys/values enter the cache in bf16,
 *     and the n_sink sink tokens and the n_recent recent ones are kept in bf16
 *     for every loop step ("Write in bf16"); for each 8 new tokens the page
 *     leaving the recent window is coded ("Encode in pages"); at step t the
 *     attention reads the coded body through slice B_t and combines it with
 *     the bf16 part ("Attend from indices").
 *   - "Results -- Long-context retrieval": n_sink = 64, n_recent = 256.
 *
 * Notation: T loop steps, Tc steps per code, NB = T/Tc code blocks,
 * H KV heads, Hq query heads (a multiple of H), D head_dim, G elements per
 * code, W = G/Tc channels per step per code, J = D/W code slots per head,
 * C <= 256 codewords (one uint8 index).  bits/element = log2(C)/G.
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  Pointers documented "device" must be
 *     device (or managed) memory of the current CUDA device; "host" pointers
 *     are ordinary host memory.  The library allocates nothing.  Its only
 *     global state is the fixed scratch array of loopvq_decode_attn_noalloc;
 *     otherwise calls on different streams are independent unless they share
 *     output, workspace or fault-word buffers.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Argument errors are detected on the host and returned
 *     before anything is launched.
 *   - Faults that only the device can see (a code >= n_codes, a context or
 *     offset outside the pools, a bounded wait that gave up) never trap: the
 *     kernel ORs a LOOPVQ_FAULT_* bit into a word in caller memory -- the
 *     workspace's status word (loopvq_read_device_status) or a fault_bits
 *     argument -- skips the offending work and finishes.
 *   - All integer sizes are element counts unless a name ends in _bytes.
 */
#ifndef LOOPVQ_H_
#define LOOPVQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LOOPVQ_API __attribute__((visibility("default")))
#else
#define LOOPVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* loopvq_stream_t;

typedef enum {
  LOOPVQ_OK = 0,
  LOOPVQ_ERR_INVALID_ARG = 1,          /* null pointer, bad size, misaligned pointer */
  LOOPVQ_ERR_UNSUPPORTED = 2,          /* valid geometry that no kernel implements */
  LOOPVQ_ERR_WORKSPACE_TOO_SMALL = 3,
  LOOPVQ_ERR_CUDA = 4,                 /* a CUDA runtime call failed (launch, attribute) */
  LOOPVQ_ERR_DEVICE_FAULT = 5          /* the device status word is non-zero */
} loopvq_status;

typedef enum { LOOPVQ_F32 = 0, LOOPVQ_BF16 = 1 } loopvq_dtype;

/* Which cache a code stream belongs to; K and V pools use different byte
 * orders inside a tile (see loopvq_index_pool_bytes). */
typedef enum { LOOPVQ_KEYS = 0, LOOPVQ_VALUES = 1 } loopvq_kind;

/* Device status word bits (see loopvq_read_device_status). */
#define LOOPVQ_FAULT_CODE_RANGE   0x1u  /* a K or V code >= n_codes was read */
#define LOOPVQ_FAULT_CTX_RANGE    0x2u  /* ctx_len > max_ctx_len or < 0 */
#define LOOPVQ_FAULT_POOL_RANGE   0x4u  /* body/window outside its pool, or misaligned body_off */
#define LOOPVQ_FAULT_TIMEOUT      0x8u  /* a bounded wait on a copy gave up (never expected) */

/*
 * One codebook family: K and V of one layer each have their own codebooks of
 * this shape.  Reading (pages silent): one codebook per (code block b, KV head
 * h, slot j); slot j covers the contiguous channels j*W .. j*W+W-1.
 */
typedef struct {
  int32_t n_loop;        /* T >= 1 */
  int32_t tc;            /* Tc >= 1, divides T and G */
  int32_t n_heads_kv;    /* H >= 1 */
  int32_t n_heads_q;     /* Hq, a positive multiple of H */
  int32_t head_dim;      /* D, a multiple of W = G/Tc */
  int32_t group_elems;   /* G, elements per code */
  int32_t n_codes;       /* C, 1..256 */
  loopvq_dtype cb_dtype; /* element type of the codebooks */
} loopvq_codebook_desc;

/*
 * Layout flag: the caller guarantees that no kernel that may still be running
 * when the decode kernel starts writes the layout arrays (ctx_len, body_off,
 * win_off, body_pages, win_head), the index pools or the codebooks.  The
 * decode kernel is always launched as a programmatic dependent of the
 * previous kernel in the stream; with this flag it starts streaming index
 * tiles before that kernel has finished.  Queries, window pools, new-token
 * rows, outputs and the workspace are touched only after it has, with or
 * without the flag (an earlier decode call of the same cache may still be
 * storing its new token into the window pool).  Without the flag nothing is
 * read before then.
 */
#define LOOPVQ_LAYOUT_STATIC_INPUTS 0x1u
/* The body lives in pages of the index pool listed by body_pages (see below)
 * instead of at body_off. */
#define LOOPVQ_LAYOUT_PAGED_BODY 0x2u
/* The recent tokens live in a ring of win_ring slots per request (see below)
 * instead of right after the sink tokens. */
#define LOOPVQ_LAYOUT_RING_WINDOW 0x4u

/*
 * Cache layout of one decode batch.  Request r has ctx_len[r] tokens, the
 * current one included.  They split (project page, "Serving in SGLang") into
 *   sink   = min(ctx, n_sink) first tokens, bf16;
 *   body   = whole pages of codes between them;
 *   recent = n_recent + ((ctx - n_sink - n_recent) mod page) last tokens, bf16;
 * a context of at most n_sink + n_recent tokens is all bf16 (sink, then recent).
 * Window pools hold, per request, the sink tokens followed by the recent
 * tokens (oldest first) at window-pool positions win_off[r] ..; index pools
 * hold the body at index-pool positions body_off[r] ...
 */
typedef struct {
  int32_t batch;              /* >= 1 */
  int32_t n_sink;             /* >= 0 (64 on the pages) */
  int32_t n_recent;           /* >= 0 (256 on the pages) */
  int32_t page;               /* >= 1 (8 on the pages) */
  int32_t max_ctx_len;        /* host-side bound on every ctx_len[r]; sizes the launch */
  uint32_t flags;             /* LOOPVQ_LAYOUT_* bits, 0 for none */
  const int32_t* ctx_len;     /* device [batch] */
  const int64_t* body_off;    /* device [batch], multiple of 32 */
  const int64_t* win_off;     /* device [batch] */
  int64_t body_pool_tokens;   /* capacity of each index pool stream, multiple of 32 */
  int64_t win_pool_tokens;    /* capacity of each window pool stream */
  /* LOOPVQ_LAYOUT_PAGED_BODY (body_off is then ignored): body token p of
   * request r sits at index-pool position
   *   body_pages[r * max_body_pages + p / body_page_tokens] * body_page_tokens
   *     + p % body_page_tokens.
   * A page id outside [0, body_pool_tokens / body_page_tokens) sets
   * LOOPVQ_FAULT_POOL_RANGE and that page is skipped. */
  const int32_t* body_pages;  /* device [batch][max_body_pages], or NULL */
  int32_t body_page_tokens;   /* a multiple of 32 (and of page) */
  int32_t max_body_pages;     /* >= ceil(max body tokens / body_page_tokens) */
  /* LOOPVQ_LAYOUT_RING_WINDOW: request r's window region starts at win_off[r]
   * with n_sink sink slots, then a ring of win_ring slots; sink token i is at
   * win_off[r] + i and recent token k (oldest first) at
   *   win_off[r] + n_sink + (win_head[r] + k) % win_ring. */
  const int32_t* win_head;    /* device [batch], or NULL */
  int32_t win_ring;           /* >= n_recent + page - 1 */
  int32_t reserved;           /* 0 */
  /* The current token's key and value at this loop step, device bf16
   * [batch][n_heads_kv][head_dim], 4-byte aligned, or NULL.  When set, the
   * decode uses them for the current token (the last window token) and also
   * stores them in its window slot -- the pages' "write in bf16" fused into
   * attention. */
  const void* new_k;
  const void* new_v;
} loopvq_cache_layout;

/* ------------------------------------------------------------------ info */

/* Library version string, e.g. "loopvq 0.1.0 sm_100a". */
LOOPVQ_API const char* loopvq_version(void);

/* Human-readable name of a status code (never NULL). */
LOOPVQ_API const char* loopvq_status_string(loopvq_status status);

/* Checks a descriptor: LOOPVQ_OK, LOOPVQ_ERR_INVALID_ARG for an inconsistent
 * one, LOOPVQ_ERR_UNSUPPORTED for a consistent geometry that the decode
 * kernels do not implement (they need J in {8, 16, 32} and W <= 16). */
LOOPVQ_API loopvq_status loopvq_validate_desc(const loopvq_codebook_desc* desc);

/* log2(n_codes) / group_elems: bits per quantized element.  Project page,
 * "Highlights": 0.5 bit (C=256, G=16) and 0.25 bit (C=256, G=32).  Returns a
 * negative value for an invalid descriptor. */
LOOPVQ_API float loopvq_bits_per_element(const loopvq_codebook_desc* desc);

/* Host helper: splits a context of ctx_len tokens into (sink, body, recent)
 * counts by the rule of loopvq_cache_layout, so that callers lay out pools the
 * way the decode kernel reads them.  Returns LOOPVQ_ERR_INVALID_ARG for
 * negative sizes, page < 1 or a NULL output. */
LOOPVQ_API loopvq_status loopvq_ctx_split(int32_t ctx_len, int32_t n_sink, int32_t n_recent, int32_t page,
                                          int32_t* sink, int32_t* body, int32_t* recent);

/* ------------------------------------------------------------- codebooks */

/*
 * Size of the packed codebook that the kernels read (0 if desc is invalid).
 * Packed form, in order: the canonical codebook as given, then per loop step t
 * the slice B_t re-laid out as [T][H][C][J][W] (code-major), all in cb_dtype.
 */
LOOPVQ_API size_t loopvq_codebook_packed_bytes(const loopvq_codebook_desc* desc);

/*
 * Packs one codebook (K or V of one layer).
 *   canonical : device, [NB][H][J][C][Tc][W] in cb_dtype; codeword c of
 *               (b, h, j) holds element (step tt, channel w) at tt*W + w,
 *               i.e. the loop-axis sub-vector of the project page's
 *               "Overview of LoopVQ" figure.
 *   packed    : device, packed_bytes >= loopvq_codebook_packed_bytes(desc),
 *               16-byte aligned.  Must not overlap canonical.
 */
LOOPVQ_API loopvq_status loopvq_codebook_pack(const loopvq_codebook_desc* desc, const void* canonical,
                                   void* packed, size_t packed_bytes, loopvq_stream_t stream);

/* ------------------------------------------------------------ index pools */

/*
 * Bytes of one index pool stream of pool_tokens tokens (K or V of one layer):
 * NB * H * pool_tokens * J, laid out [NB][H][pool_tokens/32][tile], one tile
 * = 32 tokens x J slots, one uint8 code per (token, slot); the byte order
 * inside a tile is private to the library and differs between K and V.
 * pool_tokens must be a positive multiple of 32 (else 0 is returned).
 */
LOOPVQ_API size_t loopvq_index_pool_bytes(const loopvq_codebook_desc* desc, int64_t pool_tokens);

/*
 * Writes plain codes into a pool.  codes: device [NB][H][n_tokens][J] uint8
 * (token-major, the oracle's order); they go to pool positions
 * tok_off .. tok_off+n_tokens-1 of every (b, h) stream.  Codes are stored
 * as given (no range check here; decode checks them).
 */
LOOPVQ_API loopvq_status loopvq_index_pool_pack(const loopvq_codebook_desc* desc, loopvq_kind kind,
                                     const uint8_t* codes, int64_t n_tokens,
                                     uint8_t* pool, int64_t tok_off, int64_t pool_tokens,
                                     loopvq_stream_t stream);

/* Inverse of loopvq_index_pool_pack: reads pool positions tok_off .. into
 * codes [NB][H][n_tokens][J]. */
LOOPVQ_API loopvq_status loopvq_index_pool_unpack(const loopvq_codebook_desc* desc, loopvq_kind kind,
                                       const uint8_t* pool, int64_t tok_off, int64_t pool_tokens,
                                       int64_t n_tokens, uint8_t* codes, loopvq_stream_t stream);

/* ------------------------------------------------------------------ encode */

/*
 * Loop-axis VQ encode (project page, "Component 1"): for every code block b,
 * KV head h, slot j and token n, forms the sub-vector
 *   x[tt*W + w] = X[b*Tc + tt][n][h][j*W + w],  tt < Tc, w < W
 * and stores argmin_c sum_g (x[g] - codeword_c[g])^2 over c < n_codes, ties
 * to the lowest c, at pool position tok_off + n.
 *   cb_packed : device, from loopvq_codebook_pack (this stream's kind).
 *   x         : device, element (t, n, h, d) at
 *               x[t*stride_t + n*stride_n + h*stride_h + d] in x_dtype; d is
 *               contiguous.  Strides are in elements and must be >= 0.
 *               E.g. a prefill tensor [T][N][H][D] has strides (N*H*D, H*D, D);
 *               a window pool [T][H][P][D] has (H*P*D, D, P*D).
 *   kind      : the stream written (K and V tiles differ in byte order).
 *   idx_pool  : device, loopvq_index_pool_bytes(desc, pool_tokens) bytes.
 * n_tokens = 0 is a no-op.  tok_off + n_tokens must not exceed pool_tokens.
 * Kernels: bf16 x with a bf16 256-entry codebook, G in {16, 32}, W a multiple
 * of 4, x 8-byte aligned, strides multiples of 4 and n_tokens >= 256 run on
 * the tensor cores (tcgen05: d = |x|^2 + |c|^2 - 2 x.c in fp32, with every
 * near-tie re-solved exactly from the differences); everything else runs the
 * CUDA-core kernel.  Both return the nearest codeword up to fp32 rounding of
 * distances that are equal within it.
 *   fault_bits : device uint32, 4-byte aligned, into which the kernel ORs
 *               LOOPVQ_FAULT_* bits (the caller zeroes it and reads it after
 *               the stream), or NULL to drop them.  The only fault is a
 *               bounded wait on the tensor cores that gave up (never
 *               expected): that tile's codes are left unwritten and
 *               LOOPVQ_FAULT_TIMEOUT is set.
 */
LOOPVQ_API loopvq_status loopvq_encode(const loopvq_codebook_desc* desc, const void* cb_packed,
                            loopvq_kind kind, const void* x, loopvq_dtype x_dtype,
                            int64_t n_tokens, int64_t stride_t, int64_t stride_n,
                            int64_t stride_h, uint8_t* idx_pool, int64_t tok_off,
                            int64_t pool_tokens, uint32_t* fault_bits, loopvq_stream_t stream);

/* ------------------------------------------------ codebook construction */

/*
 * One Lloyd (k-means) update of every codebook.  Project page, "Method" --
 * "Loop-aware codebook fine-tuning": the codebooks are fine-tuned against the
 * full-precision model from a start the pages do not state; the data-driven
 * start is k-means on the loop-axis sub-vectors, i.e. rounds of
 * loopvq_encode (nearest-codeword assignment) followed by this call.
 * Codeword c of (block b, head h, slot j) becomes the mean, in fp32, of the
 * sub-vectors of the n_tokens tokens whose stored code is c; a codeword no
 * token uses keeps its value from cb_in.  Codes >= n_codes are ignored.
 *   x, x_dtype, n_tokens, strides : as in loopvq_encode.
 *   kind, idx_pool, tok_off, pool_tokens : where loopvq_encode wrote the
 *               codes of these tokens (token n at pool position tok_off + n).
 *   cb_in, cb_out : device, CANONICAL layout [NB][H][J][C][Tc][W] in
 *               desc->cb_dtype (bf16 output is rounded to nearest); must not
 *               alias.  Re-pack cb_out with loopvq_codebook_pack before
 *               encoding or decoding with it.
 *   counts_out : device int32 [NB][H][J][C] member counts, or NULL.
 *   workspace  : device, 256-byte aligned, at least
 *               loopvq_codebook_update_workspace_bytes(desc) bytes; the call
 *               zeroes it on the stream.
 * Sums use fp32 atomics, so results are reproducible only up to rounding.
 */
LOOPVQ_API size_t loopvq_codebook_update_workspace_bytes(const loopvq_codebook_desc* desc);
LOOPVQ_API loopvq_status loopvq_codebook_update(const loopvq_codebook_desc* desc, loopvq_kind kind,
                                                const void* x, loopvq_dtype x_dtype, int64_t n_tokens,
                                                int64_t stride_t, int64_t stride_n, int64_t stride_h,
                                                const uint8_t* idx_pool, int64_t tok_off, int64_t pool_tokens,
                                                const void* cb_in, void* cb_out, int32_t* counts_out,
                                                void* workspace, size_t workspace_bytes, loopvq_stream_t stream);

/* ---------------------------------------------------------------- decode */

/* Workspace bytes loopvq_decode_attn needs for this layout (0 if invalid). */
LOOPVQ_API size_t loopvq_decode_workspace_bytes(const loopvq_codebook_desc* desc,
                                     const loopvq_cache_layout* layout);

/*
 * Decode attention of loop step `loop_step` for every request and query head
 * (project page, "Serving in SGLang -- Attend from indices"):
 *   o = sum_n softmax(softmax_scale * q . k_n) v_n  over the request's tokens,
 * where window tokens use the bf16 keys/values as stored and body tokens use
 *   k_n[j*W + w] = B^K_{b,h,j}[idxK[n][j]][t - b*Tc][w],  b = t / Tc
 * (and v_n likewise from idxV and B^V): the shared index row read through the
 * step's slice of the codebook.  One softmax covers window and body.
 *   cbK_packed, cbV_packed : device, packed K and V codebooks.
 *   idxK_pool, idxV_pool   : device index pools (LOOPVQ_KEYS / LOOPVQ_VALUES
 *                            byte orders), 16-byte aligned.
 *   winK, winV             : device bf16 [T][H][win_pool_tokens][D].
 *   q                      : device [batch][Hq][D] in q_dtype.
 *   out                    : device [batch][Hq][D] in out_dtype (fp32 keeps
 *                            the full accuracy; bf16 rounds the result).
 *   lse_out                : device [batch][Hq] fp32 natural-log
 *                            log-sum-exp of the scaled scores, or NULL.
 *   workspace              : device, >= loopvq_decode_workspace_bytes, 256-byte
 *                            aligned, ZERO-FILLED before its first use (it
 *                            holds the status word and the split partials);
 *                            only loopvq_clear_device_status resets the
 *                            status word.
 * Query head hq reads KV head hq / (Hq / H).  A request with ctx_len 0 gets a
 * zero output and lse -inf.  Calls sharing a workspace must be serialised
 * (same stream, or ordered by events).
 * Each call launches two kernels on `stream`, both as programmatic dependents
 * of what precedes them: the split kernel (one CTA per split of each request
 * and query head) and a merge kernel that combines the splits' partials by
 * log-sum-exp.  The layout's flags, page table, ring window and new-token
 * inputs are described with loopvq_cache_layout.
 */
LOOPVQ_API loopvq_status loopvq_decode_attn(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                 const void* cbV_packed, const loopvq_cache_layout* layout,
                                 const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                 const void* winK, const void* winV, const void* q,
                                 loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                 void* out, loopvq_dtype out_dtype, float* lse_out,
                                 void* workspace, size_t workspace_bytes,
                                 loopvq_stream_t stream);

/*
 * Several loop steps of one decode in a single launch: steps first_step ..
 * first_step + n_steps - 1, for a caller that has every step's query at once
 * (a fused all-steps decode).  This is not loop-sequential decoding, where
 * step t+1's query is computed from step t's output and each step is its own
 * loopvq_decode_attn call.  Step t of the launch computes exactly what
 * loopvq_decode_attn(loop_step = t) computes; the split kernel places the
 * CTAs of the n_steps steps that share a (query head, split) next to each
 * other, so the steps of one code block read each index row from HBM once
 * and from L2 after that.
 *   q            : device [n_steps][batch][Hq][D] in q_dtype.
 *   out, lse_out : device [n_steps][batch][Hq][D] and [n_steps][batch][Hq]
 *                  (lse_out may be NULL).
 *   workspace    : >= loopvq_decode_steps_workspace_bytes(desc, layout,
 *                  n_steps) bytes, as for loopvq_decode_attn.
 *   layout->new_k, new_v : if given, device bf16 [n_steps][batch][H][D], the
 *                  current token's K and V at each of the steps.
 * Everything else is as for loopvq_decode_attn; 1 <= n_steps and
 * first_step + n_steps <= n_loop.
 */
LOOPVQ_API size_t loopvq_decode_steps_workspace_bytes(const loopvq_codebook_desc* desc,
                                                      const loopvq_cache_layout* layout, int32_t n_steps);
LOOPVQ_API loopvq_status loopvq_decode_attn_steps(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                                  const void* cbV_packed, const loopvq_cache_layout* layout,
                                                  const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                                  const void* winK, const void* winV, const void* q,
                                                  loopvq_dtype q_dtype, int32_t first_step, int32_t n_steps,
                                                  float softmax_scale, void* out, loopvq_dtype out_dtype,
                                                  float* lse_out, void* workspace, size_t workspace_bytes,
                                                  loopvq_stream_t stream);

/*
 * Allocation-free variant of loopvq_decode_attn (the LoopVQ pages have no
 * counterpart; this is a packaging choice of the library).
 *
 * For callers that cannot allocate device memory: a plugin running inside a
 * host process whose allocator owns the GPU's memory, or a latency-critical
 * path that must not call cudaMalloc (it synchronizes the device).  Arguments
 * and results are those of loopvq_decode_attn, except that there is no
 * workspace: the split partials and counters live in a fixed 8 MiB array
 * inside the library's device image, present on every GPU that loads the
 * library until the process exits.  Nothing is allocated or freed here.
 *   fault_bits : device uint32 that receives the LOOPVQ_FAULT_* bits of this
 *                call (OR-ed in; the caller zeroes it), or NULL to drop them.
 * Returns LOOPVQ_ERR_WORKSPACE_TOO_SMALL when the layout would need more than
 * the 8 MiB array (loopvq_decode_workspace_bytes tells how much it needs).
 * The first call on a device looks up the array's device address (a
 * cudaGetSymbolAddress with that device current) and caches it for the life
 * of the process; make that first call before any stream capture, and do not
 * reset the device (cudaDeviceReset) between calls.  Every call shares the
 * one array per device: every split writes its partial before the merge
 * reads it, so nothing needs clearing, but two calls whose kernels overlap
 * on the GPU (different streams, no ordering) race on it and give wrong
 * results.
 */
LOOPVQ_API loopvq_status loopvq_decode_attn_noalloc(const loopvq_codebook_desc* desc, const void* cbK_packed,
                                                    const void* cbV_packed, const loopvq_cache_layout* layout,
                                                    const uint8_t* idxK_pool, const uint8_t* idxV_pool,
                                                    const void* winK, const void* winV, const void* q,
                                                    loopvq_dtype q_dtype, int32_t loop_step,
                                                    float softmax_scale, void* out, loopvq_dtype out_dtype,
                                                    float* lse_out, uint32_t* fault_bits,
                                                    loopvq_stream_t stream);

/* Waits for `stream`, then reads the workspace status word: LOOPVQ_OK if it
 * is zero, else LOOPVQ_ERR_DEVICE_FAULT with the LOOPVQ_FAULT_* bits stored
 * in *bits (if bits is non-NULL). */
LOOPVQ_API loopvq_status loopvq_read_device_status(const void* workspace, uint32_t* bits,
                                        loopvq_stream_t stream);

/* Zeroes the status word (asynchronously on stream). */
LOOPVQ_API loopvq_status loopvq_clear_device_status(void* workspace, loopvq_stream_t stream);

/* ------------------------------------- codebook gradient (fine-tuning) */

/*
 * Gradients of the decode-attention output error with respect to both
 * codebooks: the stand-in objective for loop-aware codebook fine-tuning
 * (project page, "Method" -- "Component 2, Loop-aware codebook fine-tuning":
 * codebooks tuned so that the quantized model's output matches the
 * full-precision one while every loop step reads the quantized cache).  At
 * loop step t,
 *   L = weight * sum_{request r, query head hq} || out[r][hq] - target[r][hq] ||^2
 * where out is loopvq_decode_attn's fp32 output of the same step, layout,
 * codes and queries, and target is, e.g., attention over the full-precision
 * cache (a per-step weight models the steps' unequal sensitivity).  With
 * g = 2 weight (o - target) and p_n = exp(s_n - lse) the softmax weight of
 * body token n, the call ADDS
 *   gradV[b][h][j][c][t-b*Tc][w] += sum_{n: idxV[n][j]=c} p_n g[j*W+w]
 *   gradK[b][h][j][c][t-b*Tc][w] += sum_{n: idxK[n][j]=c} p_n (g.v_n - g.o) scale q[j*W+w]
 * (b = t / Tc; other blocks and slices are untouched) and, if loss_out is
 * non-NULL, adds L to *loss_out.  Window tokens are bf16 and reach no
 * codebook entry (they act only through out and lse), so winK/winV are not
 * read.  Several requests of the layout may share one cache (equal body_off
 * or page tables): the gradient is then summed over their queries.
 *   cbK, cbV       : device, CANONICAL layout [NB][H][J][C][Tc][W] in
 *                    desc->cb_dtype (the values the forward's packed
 *                    codebooks were made from).
 *   layout, idxK_pool, idxV_pool, q, q_dtype, loop_step, softmax_scale : as
 *                    given to loopvq_decode_attn.
 *   out            : device fp32 [batch][Hq][D], the forward's output.
 *   lse            : device fp32 [batch][Hq], the forward's lse_out.
 *   target         : device fp32 [batch][Hq][D].
 *   gradK, gradV   : device fp32, canonical layout, accumulated into (the
 *                    caller zeroes them).
 *   loss_out       : device fp32 scalar, accumulated into, or NULL.
 *   fault_bits     : device uint32 receiving LOOPVQ_FAULT_* bits (a code
 *                    >= n_codes: that token is skipped; a context or pool
 *                    out of range: that request is skipped), or NULL.
 * J must be 8, 16 or 32 and D 64 or 128.  One kernel on `stream`; sums use
 * fp32 atomics, so results are reproducible only up to rounding order.
 */
LOOPVQ_API loopvq_status loopvq_codebook_grad(const loopvq_codebook_desc* desc, const void* cbK, const void* cbV,
                                              const loopvq_cache_layout* layout, const uint8_t* idxK_pool,
                                              const uint8_t* idxV_pool, const void* q, loopvq_dtype q_dtype,
                                              int32_t loop_step, float softmax_scale, const float* out,
                                              const float* lse, const float* target, float weight,
                                              float* gradK, float* gradV, float* loss_out,
                                              uint32_t* fault_bits, loopvq_stream_t stream);

/* ------------------------------ adjacent-loop KV-residual quantization */

/*
 * Second workload on the same loop axis (FlashLoop page, thelatestinai.com:
 * "Figure 2 (c)", "Figure 3 (c-d)", "Table 2", "Figure 4"): the K/V residual
 * between adjacent loop steps is coded with 4 bits.  Step 0 codes K_0; step t
 * codes R_t = K_t - Khat_{t-1} (the previous step's reconstruction), and
 * Khat_t = Khat_{t-1} + Q(R_t).  Q is KIVI's 4-bit asymmetric quantizer with
 * an fp16 minimum and an fp16 scale per group of 32 values: keys are grouped
 * per channel over 32 consecutive tokens, values per token over 32
 * consecutive channels (5 bits per element with the parameters).  Every
 * decision is taken in fp32 with separately rounded operations:
 *   scale = (max - min) / 15;  min_h, scale_h = fp16(min), fp16(scale)
 *   code  = scale_h == 0 ? 0 : clamp(rint((x - min_h) / scale_h), 0, 15)
 *   dequant = min_h + code * scale_h
 * Pools (pool_tokens a multiple of 32):
 *   codes       [T][H][pool_tokens][D/2] uint8, channel 2i in the low nibble
 *   key params  [T][H][pool_tokens/32][D] (min, scale) fp16 pairs
 *   value params[T][H][pool_tokens][D/32] (min, scale) fp16 pairs
 * A request's tokens start at a pool position that is a multiple of 32.
 */
typedef struct {
  int32_t n_loop;      /* T */
  int32_t n_heads_kv;  /* H */
  int32_t n_heads_q;   /* Hq, a multiple of H */
  int32_t head_dim;    /* D: 64 or 128 */
} loopvq_residual_desc;

/* Bytes of one codes pool / one parameter pool for pool_tokens tokens (0 if
 * the descriptor is invalid or pool_tokens is not a positive multiple of 32). */
LOOPVQ_API size_t loopvq_residual_codes_bytes(const loopvq_residual_desc* desc, int64_t pool_tokens);
LOOPVQ_API size_t loopvq_residual_params_bytes(const loopvq_residual_desc* desc, loopvq_kind kind,
                                               int64_t pool_tokens);

/*
 * Codes all T loop steps of n_tokens tokens of x (keys or values, element
 * (t, n, h, d) at t*stride_t + n*stride_n + h*stride_h + d, bf16 or fp32)
 * into the pools at positions tok_off .. tok_off + n_tokens - 1 (tok_off a
 * multiple of 32; a last key group shorter than 32 tokens takes its min and
 * scale over the tokens present).  One kernel on `stream`.
 */
LOOPVQ_API loopvq_status loopvq_residual_encode(const loopvq_residual_desc* desc, loopvq_kind kind, const void* x,
                                                loopvq_dtype x_dtype, int64_t n_tokens, int64_t stride_t,
                                                int64_t stride_n, int64_t stride_h, uint8_t* codes, void* params,
                                                int64_t tok_off, int64_t pool_tokens, loopvq_stream_t stream);

/* Workspace bytes of loopvq_residual_decode_attn (0 if invalid). */
LOOPVQ_API size_t loopvq_residual_decode_workspace_bytes(const loopvq_residual_desc* desc, int32_t batch,
                                                         int32_t max_ctx_len);

/*
 * Decode attention at loop step t over the residual-coded cache: request r's
 * ctx_len[r] tokens at pool positions tok_off[r] .. (every token coded, no
 * bf16 window); o = softmax(softmax_scale * q . k) v in fp32 over the key and
 * value rows that the t+1 residual planes rebuild (the encoder's
 * reconstruction).  At t = 0 the key row is rebuilt per element as the
 * encoder does; from t = 1 on q . k is taken as sum_d q_d sum_p min_p[d] plus
 * integer dot products of the codes with q_d scale_p[d] in three int8 digits
 * per 16-channel block (relative error below 2.5e-7 of the block's largest
 * weight), and values as code * scale per element plus the minima once per
 * token.  The t+1 planes of a 64-token tile must fit one shared-memory
 * stage: t+1 <= 16 at D = 128, <= 33 at D = 64 (LOOPVQ_ERR_UNSUPPORTED
 * beyond).
 *   ctx_len, tok_off : device [batch] int32 / int64.
 *   q [batch][Hq][D] in q_dtype; out [batch][Hq][D] fp32; lse_out nullable.
 *   codesK/V  : 8-byte aligned; paramsK 16-byte, paramsV 4-byte aligned.
 *   workspace : zero-filled before its first use (status word, split
 *               counters, partials), 256-byte aligned.
 * A request with ctx_len 0 gets a zero output and lse -inf; a context or
 * offset out of range sets a LOOPVQ_FAULT_* bit in the workspace status word
 * (loopvq_read_device_status) and gives that request a zero output.
 */
LOOPVQ_API loopvq_status loopvq_residual_decode_attn(const loopvq_residual_desc* desc, int32_t batch,
                                                     int32_t max_ctx_len, const int32_t* ctx_len,
                                                     const int64_t* tok_off, int64_t pool_tokens,
                                                     const uint8_t* codesK, const void* paramsK,
                                                     const uint8_t* codesV, const void* paramsV, const void* q,
                                                     loopvq_dtype q_dtype, int32_t loop_step, float softmax_scale,
                                                     float* out, float* lse_out, void* workspace,
                                                     size_t workspace_bytes, loopvq_stream_t stream);

/* -------------------------------------------------- dense bf16 comparator */

/* Workspace bytes of loopvq_dense_decode_attn. */
LOOPVQ_API size_t loopvq_dense_decode_workspace_bytes(int32_t batch, int32_t n_heads_q, int32_t head_dim,
                                           int32_t max_ctx_len);

/*
 * Plain bf16 decode attention with the same split-K structure, used as the
 * dense comparator (the pages compare against bf16 serving): every token of
 * request r is read from k/v [H][kv_pool_tokens][D] bf16 (one loop step's
 * cache) at positions kv_off[r] .. kv_off[r]+ctx_len[r]-1.
 *   q [batch][Hq][D] in q_dtype, out [batch][Hq][D] fp32, lse_out nullable.
 *   ctx_len, kv_off : device [batch] (int32, int64).
 *   workspace: zero-filled before first use, as for loopvq_decode_attn.
 * D must be 64 or 128.
 */
LOOPVQ_API loopvq_status loopvq_dense_decode_attn(int32_t batch, int32_t n_heads_kv, int32_t n_heads_q,
                                       int32_t head_dim, int32_t max_ctx_len,
                                       const int32_t* ctx_len, const int64_t* kv_off,
                                       int64_t kv_pool_tokens, const void* k, const void* v,
                                       const void* q, loopvq_dtype q_dtype, float softmax_scale,
                                       float* out, float* lse_out, void* workspace,
                                       size_t workspace_bytes, loopvq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LOOPVQ_H_ */
