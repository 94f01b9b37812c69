/*
 * hgx_attn.h -- C ABI of the hybrid-masked GQA attention core of unified text+pixel
 * transformers, for NVIDIA B200 (sm_100a).
 *
 * One call computes, for a packed batch of mixed text+image token sequences,
 *
 *   q' = rope(rmsnorm(q) * wq),  k' = rope(rmsnorm(k) * wk)      (in place, bf16)
 *   out[b, i, h] = sum_{j visible from i} softmax_j(q'[i,h] . k'[j,h/4] * scale) v[j,h/4]
 *
 * Sources (named by page title and section):
 *  - Shapes (32 query heads over 8 KV heads, head_dim 128), "q/k RMSNorm", "3-axis
 *    interleaved mRoPE [24,20,20] at theta 5e6", the sequence layout
 *    [text ... <|boi|><|tms|>] + [target patches] + [reference patches] and its mask
 *    (text causal, generation tokens see everything): "hidream-o1-p100a" model card,
 *    "What this model is".
 *  - Condition and text tokens causal, generation tokens attend to everything including
 *    the condition tokens: "HiDream-O1-Image" summary (genai-atlas), "How it works".
 *  - Generalized Causal Attention (text rows see all previous tokens; image rows see all
 *    previous tokens plus their whole image segment): "HunyuanImage 3.0 Technical Report"
 *    (paper-graph-ui summary), section 3.4, "The core rule"; bud-325 summary, "Key claims".
 *  - RoPE pairing: the half-split layout [cos(n t0), cos(n t1), ..., sin(n t0), ...] of the
 *    1D RoPE definition, same report, section 3.4, "Generalized 2D Rotary Position
 *    Embedding (RoPE)": feature k is rotated together with feature k + head_dim/2.
 *  - Rejecting bad requests before any device work: model card, "Serving (HTTP)"
 *    (contract errors return without touching the card).
 *
 * Readings where the pages are silent: softmax scale 1/sqrt(head_dim); RMSNorm eps inside
 * the square root, weight multiplies, one weight vector shared by all heads; RMSNorm
 * before RoPE; query head h reads KV head h / (Hq / Hkv); "interleaved [24,20,20]" drives
 * frequency k by axis h when k % 3 == 1 and k < 60, by axis w when k % 3 == 2 and k < 60,
 * and by axis t otherwise. HunyuanImage 3.0's Generalized 2D RoPE (same report, section
 * 3.4) is printed as [cos(x t0), cos(y t1), ...] but described as "first half x, second half
 * y"; both are offered (hgx_rope_layout), with x the w column and y the h column of pos.
 *
 * Data layout (all device tensors row-major, packed varlen: the tokens of all batch
 * elements back to back, T = cu_seqlens[batch] tokens in total):
 *   q    bf16 [T, 32, 128]  (token stride 8192 B)      -- overwritten with q'
 *   k    bf16 [T, 8, 128]   (token stride 2048 B)      -- overwritten with k'
 *   v    bf16 [T, 8, 128]                               -- read only
 *   out  bf16 [T, 32, 128]                              -- written
 *   pos  int32 [T, 3]  (t, h, w) position of each token -- read only
 *   wq, wk bf16 [128]  RMSNorm weights                  -- read only
 * Every device pointer must be non-null (when T > 0) and 16-byte aligned; out must not
 * overlap q, k or v. V must be finite within each batch element: a row's masked
 * probabilities (exact zeros) meet V rows of its own element that it cannot see, and
 * 0 * inf is NaN. V rows of other batch elements never reach a row's output: where a
 * 128-key block runs past the end of an element, the kernel zeroes the next element's V
 * rows in shared memory before the P V product.
 *
 * Segments: for batch element b, segs[cu_segs[b] .. cu_segs[b+1]) describe its tokens in
 * order. Each has a start local to the element, a length >= 1 and a kind. They must tile
 * [0, L_b) exactly, L_b = cu_seqlens[b+1] - cu_seqlens[b]. An element with L_b == 0 has
 * no segments. Visibility of key j from query i (both local):
 *   HGX_SEG_CAUSAL           j <= i
 *   HGX_SEG_FULL_SEQUENCE    every j < L_b
 *   HGX_SEG_FULL_IN_SEGMENT  j <= i, or j inside i's own segment
 *   HGX_SEG_GEN_IMAGE        as FULL_IN_SEGMENT for its own rows; in addition its keys are
 *                            hidden from every row of a LATER segment (the multi-Gen-Image
 *                            training mask of HunyuanImage 3.0: paper-graph-ui summary,
 *                            section 3.4, "The multi-generation training complication",
 *                            Figure 4(b))
 * Under the first three kinds the visible keys of a row form a prefix [0, lim(i)); a
 * gen_image segment cuts a hole out of the prefix of every later row.
 *
 * Ownership and threading: the caller owns every tensor and the stream. The handle owns
 * the planner's device scratch (per-row key limits, the work list, a device error word)
 * and reuses it while the segment descriptor is unchanged. A handle serves one stream at a
 * time and is not thread-safe; calls on one handle must not overlap on the GPU unless they
 * share a stream. Device calls are asynchronous on `stream` (a cudaStream_t, NULL for the
 * legacy default stream).
 *
 * Errors: every export returns hgx_status. Descriptor and pointer checks run on the host
 * before any device work; on failure nothing is launched and hgx_attn_last_error() gives a
 * message. CUDA launch failures return HGX_ERR_CUDA. Every wait inside the attention kernel
 * is bounded in time; a wait that runs out sets a device error word and the kernel returns
 * early. hgx_attn_sync_status() (called automatically in checked mode) synchronizes the
 * stream and reports that as HGX_ERR_TIMEOUT.
 */
#ifndef HGX_ATTN_H
#define HGX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HGX_OK = 0,
  HGX_ERR_INVALID_ARG = 1, /* malformed descriptor, null or misaligned pointer, bad size */
  HGX_ERR_UNSUPPORTED = 2, /* valid request outside what this build implements (shapes) */
  HGX_ERR_OOM = 3,         /* device or pinned host allocation for the planner failed */
  HGX_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
  HGX_ERR_TIMEOUT = 5      /* a bounded device wait ran out (see hgx_attn_sync_status) */
} hgx_status;

typedef enum {
  HGX_SEG_CAUSAL = 0,
  HGX_SEG_FULL_SEQUENCE = 1,
  HGX_SEG_FULL_IN_SEGMENT = 2,
  HGX_SEG_GEN_IMAGE = 3
} hgx_seg_kind;

typedef enum { HGX_TILE_SKIP = 0, HGX_TILE_PARTIAL = 1, HGX_TILE_FULL = 2 } hgx_tile_class;

typedef struct {
  int32_t start; /* first token, local to the batch element */
  int32_t len;   /* >= 1 */
  int32_t kind;  /* hgx_seg_kind */
} hgx_segment;

typedef enum {
  HGX_ROPE_MROPE_INTERLEAVED = 0, /* 3-axis (t, h, w) interleaved over mrope_section */
  HGX_ROPE_2D_ALTERNATING = 1,    /* 2D (x = w, y = h): frequency k by x if k even, else y */
  HGX_ROPE_2D_HALVES = 2          /* 2D: frequencies k < head_dim / 4 by x, the rest by y */
} hgx_rope_layout;

typedef struct {
  int32_t num_q_heads;      /* must be 32 */
  int32_t num_kv_heads;     /* must be 8 */
  int32_t head_dim;         /* must be 128 */
  double rope_theta;        /* > 0; 5e6 in the model card */
  int32_t mrope_section[3]; /* (t, h, w) frequency counts, sum head_dim / 2; {24, 20, 20} */
  float rms_eps;            /* >= 0; 1e-6 */
  float softmax_scale;      /* > 0, or 0 for 1 / sqrt(head_dim) */
  int32_t rope_layout;      /* hgx_rope_layout; mrope_section applies to the interleaved one */
} hgx_attn_config;

typedef struct hgx_attn_handle hgx_attn_handle;

/* Fills *cfg with the model card's constants (32/8/128, theta 5e6, [24,20,20], eps 1e-6,
 * scale 0 = 1/sqrt(128)). */
void hgx_attn_default_config(hgx_attn_config* cfg);

/* Validates *cfg and creates a handle. No device memory is allocated until the first
 * device call. Errors: INVALID_ARG (null, bad values), UNSUPPORTED (other shapes), OOM. */
hgx_status hgx_attn_create(const hgx_attn_config* cfg, hgx_attn_handle** out);

/* Frees the handle and its device scratch. Waits for nothing: the caller must make sure
 * no call on the handle is still running on the GPU. NULL is ignored. */
void hgx_attn_destroy(hgx_attn_handle* h);

/* Message of the last failed call on this handle ("" if none). Valid until the next call. */
const char* hgx_attn_last_error(const hgx_attn_handle* h);

/* The whole path: prologue (RMSNorm + mRoPE of q and k, in place), then masked GQA
 * attention into out. cu_seqlens_host int32 [batch+1] with cu_seqlens_host[0] == 0, and
 * segs_host / cu_segs_host (int32 [batch+1]) live in host memory and may be reused by the
 * caller as soon as the call returns. T == 0 returns HGX_OK without device work. */
hgx_status hgx_attn_forward(hgx_attn_handle* h, void* stream, void* q, void* k, const void* v,
                            void* out, const int32_t* pos_thw, const void* q_norm_w,
                            const void* k_norm_w, int32_t batch, const int32_t* cu_seqlens_host,
                            const hgx_segment* segs_host, const int32_t* cu_segs_host);

/* One denoising step with a reused prefix (the text before <|tms|> of the HiDream-O1
 * layout is causal, so its keys, values and outputs are the same in all 100 forwards of an
 * image: "hidream-o1-p100a" model card, "What this model is" and "Performance"). Only rows
 * [first_rows_host[b], L_b) of element b are computed: their q and k get the prologue,
 * their out rows are written. Rows before first_rows_host[b] keep their out, and their k
 * must already hold k' (e.g. from an earlier call); their q is not read. Every reused row
 * must see no key at or after first_rows_host[b] (HGX_ERR_INVALID_ARG otherwise). Other
 * arguments as hgx_attn_forward; first_rows_host int32 [batch], host. */
hgx_status hgx_attn_forward_from(hgx_attn_handle* h, void* stream, void* q, void* k,
                                 const void* v, void* out, const int32_t* pos_thw,
                                 const void* q_norm_w, const void* k_norm_w, int32_t batch,
                                 const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                                 const int32_t* cu_segs_host, const int32_t* first_rows_host);

/* The prologue alone on total_tokens tokens (q and k overwritten with q' and k'). */
hgx_status hgx_attn_prologue(hgx_attn_handle* h, void* stream, void* q, void* k,
                             const int32_t* pos_thw, const void* q_norm_w, const void* k_norm_w,
                             int32_t total_tokens);

/* The attention alone, on q and k that already hold q' and k' (nothing is overwritten). */
hgx_status hgx_attn_attention(hgx_attn_handle* h, void* stream, const void* q, const void* k,
                              const void* v, void* out, int32_t batch,
                              const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                              const int32_t* cu_segs_host);

/* ---------------------------------------------------------------------------------------
 * The attention layer around the core: the QKV projection in front of it and the output
 * projection behind it. Sizes from "hidream-o1-p100a" model card, "What this model is":
 * hidden size 4096, 32 query heads over 8 KV heads at head_dim 128, so the projection
 * maps 4096 features to 32*128 + 2*8*128 = 6144 and the output projection 4096 -> 4096.
 * Weights are row-major [out, in] bf16 (y = x W^T):
 *   w_qkv  bf16 [6144, 4096]: rows 0..4095 the 32 query heads (128 rows each, head h at
 *          rows 128h..128h+127), rows 4096..5119 the 8 key heads, rows 5120..6143 the 8
 *          value heads
 *   w_o    bf16 [4096, 4096]: column 128h + d reads feature d of query head h
 *   x      bf16 [T, 4096] hidden states; attn bf16 [T, 32, 128]; y bf16 [T, 4096]
 * All pointers device, non-null and 16-byte aligned; T = total_tokens <= 2^19 - 1. The
 * GEMMs run on the tensor cores with fp32 accumulation and round to bf16. */

/* q' = rope(rmsnorm(x Wq^T) * wq), k' = rope(rmsnorm(x Wk^T) * wk), v = x Wv^T: the
 * projection with the prologue's RMSNorm and rotation fused into its epilogue (no q/k
 * round trip through memory). q [T,32,128], k and v [T,8,128] are written; positions and
 * norm weights as in hgx_attn_forward. Errors: INVALID_ARG (pointer, size), CUDA, OOM
 * (the per-call (cos, sin) table of the rotation is allocated by the handle). */
hgx_status hgx_attn_qkv_projection(hgx_attn_handle* h, void* stream, const void* x,
                                   const void* w_qkv, void* q, void* k, void* v,
                                   const int32_t* pos_thw, const void* q_norm_w,
                                   const void* k_norm_w, int32_t total_tokens);

/* y = attn W_o^T, attn read as [T, 4096]. Errors: INVALID_ARG (pointer, size), CUDA. */
hgx_status hgx_attn_out_projection(hgx_attn_handle* h, void* stream, const void* attn,
                                   const void* w_o, void* y, int32_t total_tokens);

/* The whole layer: hgx_attn_qkv_projection into q, k, v, masked attention into attn
 * (segment descriptor as in hgx_attn_forward), hgx_attn_out_projection into y. q, k, v
 * and attn are caller-provided intermediates; attn must not overlap q, k or v. */
hgx_status hgx_attn_layer_forward(hgx_attn_handle* h, void* stream, const void* x,
                                  const void* w_qkv, const void* w_o, void* q, void* k, void* v,
                                  void* attn, void* y, const int32_t* pos_thw,
                                  const void* q_norm_w, const void* k_norm_w, int32_t batch,
                                  const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                                  const int32_t* cu_segs_host);

/* Host only (no GPU needed). Exclusive key limit lim(i) of every packed row, local to its
 * batch element: row i sees keys [0, lim(i)) minus the keys of gen_image segments before
 * its own segment. lim_out has room for cap entries; T entries are written. Errors:
 * INVALID_ARG (descriptor, or cap < T). */
hgx_status hgx_attn_row_limits(int32_t batch, const int32_t* cu_seqlens_host,
                               const hgx_segment* segs_host, const int32_t* cu_segs_host,
                               int32_t* lim_out, size_t cap);

/* Host only. Tile classes at the attention kernel's real tile size: *bm_tokens query
 * tokens (shared by all 4 query heads of a KV head) x *bn_keys keys. For each batch
 * element in order, ceil(L/bm) x ceil(L/bn) bytes, row-major over (query block, key
 * block), each an hgx_tile_class. Keys past the element's end count as masked, so a
 * ragged last key block is never FULL. *n_written receives the number of bytes; if
 * classes_out is NULL only the sizes are returned. */
hgx_status hgx_attn_classify(int32_t batch, const int32_t* cu_seqlens_host,
                             const hgx_segment* segs_host, const int32_t* cu_segs_host,
                             int32_t* bm_tokens, int32_t* bn_keys, uint8_t* classes_out,
                             size_t cap, size_t* n_written);

/* Host only. Number of visible (query, key) pairs of the whole packed batch (holes
 * excluded): the attention performs 4 * head_dim * num_q_heads FLOPs per pair. */
hgx_status hgx_attn_visible_pairs(int32_t batch, const int32_t* cu_seqlens_host,
                                  const hgx_segment* segs_host, const int32_t* cu_segs_host,
                                  uint64_t* pairs);

/* Host only. The schedule of the attention kernel's persistent CTAs for this descriptor on
 * `ctas` CTAs (the library uses the device's SM count), for tests and tools: 8 int32 per
 * work item in execution order, (cta, q0, kv_head, kb0, n_total, part, n_full, list_off).
 * A work item covers 64 query tokens x the 4 query heads of one KV head; it processes key
 * blocks kb0 .. kb0 + n_total - 1 (prefix form, list_off < 0) or the n_total blocks of its
 * key-block list (list form). part >= 0 marks one of the parts of a split item (slots of
 * one item are consecutive), which write partial results that a combine kernel merges.
 * mode 0: the library's own policy; 1: the CTAs loaded above the mean hand their last items
 * out in parts to the least-loaded CTAs whenever that lowers the makespan by more than the
 * combine's cost; 2: as under HGX_DEBUG_SPLIT_TEST (every prefix-form item of two or more
 * key blocks split in two). out has room for cap items (8 int32 each);
 * *n_items receives the count; out may be NULL to query the count. */
hgx_status hgx_attn_schedule(int32_t batch, const int32_t* cu_seqlens_host,
                             const hgx_segment* segs_host, const int32_t* cu_segs_host,
                             int32_t ctas, int32_t mode, int32_t* out, size_t cap,
                             size_t* n_items);

/* Synchronizes `stream`, then reads and clears the handle's device error word: returns
 * HGX_ERR_TIMEOUT if a bounded wait ran out since the last check, HGX_ERR_CUDA if the
 * stream reports an error, HGX_OK otherwise. */
hgx_status hgx_attn_sync_status(hgx_attn_handle* h, void* stream);

/* Clock of the last attention launch made through h (hgx_attn_forward, _forward_from,
 * _attention or _layer_forward); the pages have no counterpart, this is measurement. Every
 * persistent CTA of the attention kernel stamps the SM's cycle counter (clock64) and the
 * global nanosecond timer at its start and at its end into a small device buffer that the
 * handle owns. This call synchronizes `stream`, copies the stamps and returns: *cycles =
 * the largest CTA's cycle count, *ns = the largest CTA's span in nanoseconds, *sm_mhz =
 * the median over CTAs of cycles / ns (the effective SM clock, which under the power cap
 * can sit well below the clock NVML reports). HGX_ERR_INVALID_ARG if a pointer is NULL or
 * no attention kernel has run on this handle; the call does not clear the error word. */
hgx_status hgx_attn_kernel_clock(hgx_attn_handle* h, void* stream, uint64_t* cycles, uint64_t* ns,
                                 double* sm_mhz);

/* Debug flags for hgx_attn_set_debug. */
#define HGX_DEBUG_CHECKED 1u    /* every device call ends with hgx_attn_sync_status */
#define HGX_DEBUG_STALL_TEST 2u /* attention: one softmax warpgroup first waits on a barrier
                                   that nothing arrives at, so its bounded wait runs out */
#define HGX_DEBUG_FAIL_ALLOC 4u /* the next device allocation of the planner scratch reports
                                   HGX_ERR_OOM instead of allocating (one-shot: the flag
                                   clears itself); nothing is launched by that call */
#define HGX_DEBUG_SPLIT_TEST 8u /* the planner splits every prefix-form work item of two or
                                   more key blocks into two halves by key blocks (exercises
                                   the split path and its combine kernel on any input) */

/* Sets debug flags and the bound of every device wait in nanoseconds (0 keeps the
 * default of 2 s). The HGX_DEBUG environment variable (an integer) sets the initial
 * flags of new handles. */
hgx_status hgx_attn_set_debug(hgx_attn_handle* h, uint32_t flags, uint64_t wait_limit_ns);

/* ---------------------------------------------------------------------------------------
 * Allocation-free variant of hgx_attn_forward. The paper has no counterpart to this entry
 * point; it exists for callers that cannot allocate memory: code inside a framework that
 * owns all device memory through its own pool and forbids cudaMalloc behind its back, or a
 * process whose device footprint must not grow after start-up. It needs no handle (creating
 * one allocates) and calls no cudaMalloc, cudaFree, cudaMallocHost or heap allocation.
 *
 * Scratch (per-row key limits, work list, per-CTA item offsets, error word) lives in one
 * fixed-size device array inside the library (about 185 KB, held by every GPU that loads
 * the library until the process exits); planning uses fixed-size static host buffers. Hence
 * the limits: at most HGX_NOALLOC_MAX_TOKENS packed tokens and HGX_NOALLOC_MAX_BATCH batch
 * elements, and no gen_image segments; other requests return HGX_ERR_UNSUPPORTED before
 * any device work. Work items are assigned to the persistent CTAs as in hgx_attn_forward
 * (largest planned cost first, each to the least-loaded CTA).
 *
 * Arguments are those of hgx_attn_forward with the config in place of a handle (validated
 * on every call), plus `synchronize`: when nonzero the call waits for the stream and returns
 * HGX_ERR_TIMEOUT if a bounded device wait ran out; when zero it returns after the launches
 * and such a timeout goes unreported. The first call on each device looks up the device
 * address of the scratch array (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture. The plan is uploaded with cudaMemcpyAsync from the
 * library's static pageable host buffers (the driver stages each copy before the call
 * returns, so the call may wait on the host). A call on a stream that is being captured
 * (or on the legacy stream while another stream is captured) returns HGX_ERR_UNSUPPORTED
 * before any device work: a recorded copy would read those shared host buffers again at
 * replay, after later calls had rewritten them. All calls share the scratch and the host
 * buffers, which keep the previous call's contents (the error word is cleared at the start
 * of each call): calls that overlap on the GPU, or run from several host threads at once,
 * race. */
#define HGX_NOALLOC_MAX_TOKENS 16384
#define HGX_NOALLOC_MAX_BATCH 64

hgx_status hgx_attn_forward_noalloc(const hgx_attn_config* cfg, void* stream, void* q, void* k,
                                    const void* v, void* out, const int32_t* pos_thw,
                                    const void* q_norm_w, const void* k_norm_w, int32_t batch,
                                    const int32_t* cu_seqlens_host, const hgx_segment* segs_host,
                                    const int32_t* cu_segs_host, int32_t synchronize);

#ifdef __cplusplus
}
#endif

#endif /* HGX_ATTN_H */
