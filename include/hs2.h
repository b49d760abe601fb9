/*
 * hs2.h -- C ABI of libhs2: HySparse2 Cross-Decoder Hybrid-Block decode
 * attention on NVIDIA B200 (sm_100a).
 *
 * The method (HySparse2 announcement for MiMo-V3, "KV Reuse" section and the
 * two paragraphs after it on token-level selection and the forced window):
 * a Hybrid Block is one full-attention layer followed by sparse-attention
 * layers.  The full layer attends over the whole shared KV cache and, in the
 * same computation, picks important positions from its attention scores; the
 * sparse layers reuse that KV cache and that index list directly.  Selection
 * is per token: the most recent 128 tokens are always kept, plus 1,024 global
 * tokens from outside that window, and both parts are read from the one
 * shared cache in a single sparse-attention computation.
 *
 * Readings fixed where the pages are silent:
 *   score[t] of a KV head = sum over the query heads of its GQA group of the
 *   full layer's softmax probability at t; the global part is the top
 *   k_global of t < T - window by (score desc, position asc), or all such t
 *   when there are no more than k_global; query head h uses KV head
 *   floor(h / G); the softmax scale is 1/sqrt(head_dim); the current token's
 *   K/V are already in the cache at position T-1.
 *
 * Conventions for every call:
 *   - All pointers named "device" are CUDA device pointers on the current
 *     device; the library never allocates, frees or keeps any of them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream): no host synchronisation, no device-wide state.
 *   - Return value: HS2_OK or an error code; on error nothing was launched
 *     (except HS2_ERR_CUDA, where a launch itself failed) and
 *     hs2_last_error() describes the problem.
 *   - Device-side waits are bounded; an expired wait sets a sticky flag in the
 *     workspace that hs2_workspace_status() reports as HS2_ERR_TIMEOUT.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HS2_OK 0
#define HS2_ERR_INVALID_ARG 1  /* null pointer, bad shape, mismatched descriptors */
#define HS2_ERR_UNSUPPORTED 2  /* dtype / head_dim / group / page size not built */
#define HS2_ERR_WORKSPACE 3    /* workspace missing, too small or misaligned */
#define HS2_ERR_CUDA 4         /* a CUDA runtime call or a launch failed */
#define HS2_ERR_TIMEOUT 5      /* a bounded device-side wait expired */

/* Element types. */
#define HS2_F32 0  /* IEEE fp32 */
#define HS2_BF16 1 /* bfloat16 */
#define HS2_E4M3 2 /* OCP FP8 E4M3 ("fn": no inf, S.1111.111 = NaN), per-row fp32 scale */

/*
 * One K or V cache of the full layer (the cache every layer of the Hybrid
 * Block reads).  Rows are [num_slots, num_kv_heads, head_dim], row-major,
 * element type `dtype`.  Position t of sequence b lives in slot
 *     page_table[b * max_pages + t / page_size] * page_size + t % page_size
 * or, when the call's page_table is NULL (contiguous layout),
 *     b * page_size + t         (page_size = per-sequence capacity).
 * For HS2_E4M3 the stored value is decode(code) * scale[slot * num_kv_heads + h].
 */
typedef struct {
  const void *data;    /* device; 16-byte aligned */
  const float *scale;  /* device, [num_slots, num_kv_heads]; HS2_E4M3 only, else NULL */
  int32_t dtype;       /* HS2_F32, HS2_BF16 or HS2_E4M3 */
  int32_t num_kv_heads;
  int32_t head_dim;    /* 64 or 128 */
  int32_t page_size;   /* tokens per page (16, 32 or a multiple of 64 for
                          HS2_BF16/HS2_E4M3; any >= 1 for HS2_F32) */
  int64_t num_slots;   /* rows in the cache, < 2^31 */
} hs2_cache;

/* Per-head query or output vectors: [batch, num_heads, head_dim], row-major. */
typedef struct {
  void *data;          /* device; 16-byte aligned */
  int32_t dtype;       /* HS2_F32 (with an HS2_F32 cache) or HS2_BF16 */
  int32_t batch;
  int32_t num_heads;   /* num_kv_heads * G, G in {1, 2, 4, 8, 16, 32} (above 8: bf16 / E4M3 caches) */
  int32_t head_dim;
} hs2_heads;

/*
 * Bytes of workspace hs2_full_attn_select() needs for this shape on the
 * current device; t_cap = max_pages * page_size (paged) or page_size
 * (contiguous).  Returns 0 for invalid shapes.
 */
size_t hs2_full_attn_select_workspace(int32_t batch, int32_t num_kv_heads, int32_t group,
                                      int32_t head_dim, int64_t t_cap);

/*
 * Full-attention layer of a Hybrid Block, with token selection.
 *
 * Passage: HySparse2 announcement for MiMo-V3, "KV Reuse" section -- the
 * block's one full-attention layer attends over the whole shared KV cache and,
 * while computing its own attention, picks the important positions from its
 * attention scores (no separately trained selector); the next two paragraphs
 * make the selection per token and fix the budget: the most recent 128 tokens
 * always, plus 1,024 global tokens from outside that window.  (The same
 * section is 02-03 of the Vietnamese translation of the announcement.)
 *
 *   q          [B, Hq, d] device, the full layer's query of the new token.
 *   k_cache,
 *   v_cache    the shared cache (same dtype, heads, head_dim, page_size,
 *              num_slots); the current token's K/V already at position T_b-1.
 *   seq_lens   device int32 [B]: T_b, clamped to [0, t_cap] on the device.
 *   page_table device int32 [B, max_pages], or NULL for the contiguous layout
 *              (then max_pages must be 1).  Entries past ceil(T_b/page_size)
 *              are never read.
 *   window     W >= 0 (the pages use 128), k_global K >= 0 (the pages use
 *              1,024), W + K >= 1.
 *   out        [B, Hq, d] device, dtype of q: softmax(q k^T / sqrt(d)) v over
 *              all T_b positions, per query head (zeros when T_b = 0).
 *   idx_out    device int32 [B, Hkv, W + K]: for each (b, kv head) the
 *              selected positions as SLOTS (page table applied), in
 *              ascending position order, min(T_b, W + K) valid entries, the
 *              rest -1.  This is the index list every sparse layer reuses.
 *   workspace  device scratch of at least hs2_full_attn_select_workspace()
 *              bytes, 256-byte aligned, owned by the caller; its contents
 *              need no initialisation and are overwritten (except the sticky
 *              error flag).  One workspace must not serve two calls that
 *              run concurrently.
 * Limits: W + K <= 4096 (else HS2_ERR_INVALID_ARG); batch <= 4096, a
 * capacity t_cap <= 2^23 positions per sequence and
 * B * ceil(t_cap / 16) * Hkv < 2^31 (else HS2_ERR_UNSUPPORTED).
 */
int hs2_full_attn_select(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                         const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                         int32_t window, int32_t k_global, hs2_heads *out, int32_t *idx_out,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * hs2_full_attn_select() that also records `mark_event` (a cudaEvent_t, or
 * NULL) on `stream` between the attention kernel and the selection kernels,
 * so a caller can time the two parts with events.  Same arguments, same
 * results.
 */
int hs2_full_attn_select_marked(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                                const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                                int32_t window, int32_t k_global, hs2_heads *out, int32_t *idx_out,
                                void *workspace, size_t workspace_bytes, void *stream, void *mark_event);

/*
 * hs2_full_attn_select() as one fused persistent pass: the attention kernel's
 * CTAs, after their last tile, wait at a grid barrier and run the selection's
 * score pass over the positions they attended (logits still in L2), so the
 * full layer selects as it finishes its own computation (HySparse2
 * announcement, "KV Reuse" section: the full layer's attention scores pick
 * the positions the sparse layers read).  Same arguments and results as
 * hs2_full_attn_select(); two more kernels (filter, final) follow on `stream`.
 *   The kernel is launched cooperatively (every CTA resident at once; no
 *   programmatic overlap with the previous kernel); the call first clears
 *   the barrier's counter with cudaMemsetAsync.  The barrier wait is bounded
 *   (about 2 s): on expiry the sticky flag reports HS2_ERR_TIMEOUT through
 *   hs2_workspace_status() and the selection of that call is not valid.
 *   Tensor-core caches (bf16, E4M3) in the default configuration of their
 *   shape only; fp32 caches run the unfused call.  HS2_ERR_UNSUPPORTED for
 *   shapes with no fused kernel built.
 */
int hs2_full_attn_select_fused(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                               const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                               int32_t window, int32_t k_global, hs2_heads *out, int32_t *idx_out,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * The full-attention layer with BLOCK-level instead of token-level selection:
 * the first-generation HySparse selection, kept as a comparator (HySparse2
 * announcement, the paragraphs contrasting token-level with HySparse's
 * block-level selection: v1 chose whole blocks, so an important token brought
 * the block around it; the two were compared at the same token budget).
 * Readings: the selectable positions [0, T_b - W) are cut into blocks of
 * `block` positions, the last one cut short at T_b - W; a block's score is
 * the sum of its positions' group scores (as for hs2_full_attn_select());
 * k_global / block blocks are taken by (block score desc, block index asc),
 * all of them when there are no more; the window is always taken.
 *
 *   Arguments as hs2_full_attn_select(), plus block >= 1 dividing k_global
 *   (else HS2_ERR_INVALID_ARG).  out is the same attention output; idx_out
 *   holds the slots of the taken positions in ascending position order (the
 *   taken blocks' positions, then the window), the rest -1.  The workspace is
 *   that of hs2_full_attn_select() (same size function).
 */
int hs2_full_attn_select_blocks(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                                const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                                int32_t window, int32_t k_global, int32_t block, hs2_heads *out, int32_t *idx_out,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * hs2_full_attn_select() for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for integration.
 *
 * Some callers only receive device pointers and a stream and are not allowed
 * to call cudaMalloc: a plugin inside a serving engine that has reserved
 * nearly all HBM for its own KV-cache pool up front, or an extension of a
 * runtime that plans every buffer before execution and gives its kernels no
 * scratch.  They cannot provide the workspace hs2_full_attn_select() needs,
 * so this call uses a scratch array that the library itself owns: a fixed
 * 32 MiB device array that every GPU which loads the library keeps until the
 * process exits.  The call allocates nothing.
 *
 *   Arguments and results are those of hs2_full_attn_select() without the
 *   workspace.  Shapes whose workspace (hs2_full_attn_select_workspace())
 *   exceeds 32 MiB are rejected with HS2_ERR_WORKSPACE and a message.
 *   The first call in each CUDA context (per device, for the runtime's primary
 *   contexts) looks up the array's device address in that context; make that
 *   first call before any stream capture begins.
 *   All calls share the one array and it keeps the last call's contents (the
 *   kernels clear what must start at zero themselves): calls that overlap on
 *   the GPU -- on different streams, or from different threads -- race and
 *   must be serialised by the caller.
 *   Word 0 of the array is the sticky device-error flag of these calls; read
 *   it with hs2_full_attn_select_static_status().
 */
int hs2_full_attn_select_static(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                                const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                                int32_t window, int32_t k_global, hs2_heads *out, int32_t *idx_out,
                                void *stream);

/*
 * Status of hs2_full_attn_select_static() calls in the current CUDA context
 * (no counterpart in the pages): synchronises `stream`, then reads and clears
 * the static scratch's sticky device-error flag.  HS2_OK, or HS2_ERR_TIMEOUT
 * if a bounded device wait of an earlier static call expired (its out and
 * idx_out are then incomplete).
 */
int hs2_full_attn_select_static_status(void *stream);

/*
 * Passage: HySparse2 announcement, "KV Reuse" section and the paragraph after
 * the forced window -- every sparse layer of the block reuses the full
 * layer's KV cache and its selection indices directly, and reads the window
 * and the global tokens from that one cache in a single sparse-attention
 * computation, with no sliding-window branch and no KV cache of its own.
 *
 * Sparse-attention layer of a Hybrid Block: for each (b, query head h) the
 * softmax of q_l k^T / sqrt(d) over the rows idx[b, floor(h/G), :] (slots,
 * -1 entries skipped), times those V rows.  It reads the same shared cache as
 * the full layer and the index list that hs2_full_attn_select() wrote; its
 * query q_l is the layer's own.  A (b, head) with no valid row gets zeros.
 *
 *   idx        device int32 [B, Hkv, idx_stride], idx_stride in [1, 4096].
 *   out        [B, Hq, d] device, dtype of q_l.
 * Needs no workspace.
 */
int hs2_sparse_attn(const hs2_heads *q_l, const hs2_cache *k_cache, const hs2_cache *v_cache,
                    const int32_t *idx, int32_t idx_stride, hs2_heads *out, void *stream);

/*
 * Synchronises `stream`, then reads and clears the workspace's sticky
 * device-error flag: HS2_OK, or HS2_ERR_TIMEOUT if a bounded device wait of
 * an earlier call on this workspace expired.
 */
int hs2_workspace_status(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Device-to-device copy of `bytes` (a multiple of 16, both pointers 16-byte
 * aligned) with a grid sized to the SM count: the HBM copy-bandwidth
 * reference that the roofline is quoted against.
 */
int hs2_copy_peak(void *dst, const void *src, size_t bytes, void *stream);

/* Thread-local text of the last non-zero status returned on this thread. */
/*
 * Workspace bytes of hs2_kv_bridge_append() for this shape (0 if invalid).
 */
size_t hs2_kv_bridge_workspace(int32_t batch, int32_t d_model, int32_t num_kv_heads, int32_t head_dim);

/*
 * KV Bridging append of one decode step (HySparse2 announcement, "KV
 * Bridging" paragraphs): each Cross-Decoder full-attention layer builds its
 * own KV cache from the input hidden state of the matching Self-Decoder
 * full-attention layer, through its own K and V projections.  For every
 * sequence b the new token's rows
 *     k_b = h_b W_k,   v_b = h_b W_v          (fp32 accumulation, no bias)
 * are written at position T_b - 1 (the token being decoded, already counted in
 * seq_lens, as hs2_full_attn_select() expects) of k_cache / v_cache through
 * the page table: as computed for HS2_F32, rounded to nearest even for
 * HS2_BF16, and for HS2_E4M3 with scale = max_i |x_i| / 448 per (token, kv
 * head) (1 for an all-zero row) and codes the E4M3 values nearest x / scale
 * (ties to even), saturated at +-448.
 *
 *   hidden     device bf16 [batch, d_model], 16-byte aligned; d_model a
 *              positive multiple of 128.
 *   w_k, w_v   device bf16 [d_model, num_kv_heads * head_dim], row-major,
 *              16-byte aligned (the layer's own projections).
 *   seq_lens   device int32 [batch]: T_b, clamped to [0, t_cap]; T_b = 0
 *              writes nothing.
 *   page_table device int32 [batch, max_pages], or NULL (contiguous layout,
 *              max_pages = 1).  A page outside the cache writes nothing.
 *   k_cache,
 *   v_cache    the caches to write (descriptors as for hs2_full_attn_select;
 *              this call writes one row per (sequence, kv head) and, for
 *              E4M3, its scale).
 *   workspace  device, >= hs2_kv_bridge_workspace() bytes, 256-byte aligned,
 *              zero-filled before its first use: it starts with one counter
 *              per (K or V, 128-column tile, group of 8 sequences) that the
 *              call's last CTA of each returns to zero, so a workspace is
 *              reused as is; calls sharing one must not overlap on the GPU.
 * Asynchronous on `stream`; rows of other positions are not touched.  The
 * result does not depend on the order in which CTAs finish.
 */
int hs2_kv_bridge_append(const void *hidden, int32_t batch, int32_t d_model, const void *w_k, const void *w_v,
                         const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                         const hs2_cache *k_cache, const hs2_cache *v_cache, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Self-test of the bounded device waits (no counterpart in the pages): one
 * CTA waits on a barrier that nothing completes; the wait gives up after
 * about 10 ms of clock cycles and sets the workspace's sticky flag, so a
 * following hs2_workspace_status() returns HS2_ERR_TIMEOUT (and clears it)
 * and the CUDA context stays usable.  No fault, trap or hang is involved.
 *   workspace  device, >= 256 bytes, 256-byte aligned (only its flag word is used).
 * Returns HS2_OK once launched (asynchronous on `stream`).
 */
int hs2_selftest_bounded_wait(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Self-test of the fused call's grid barrier (no counterpart in the pages):
 * two CTAs meet at a barrier sized for three, both give up after about 10 ms
 * of clock cycles and set the workspace's sticky flag (bit 8), so a
 * following hs2_workspace_status() returns HS2_ERR_TIMEOUT (and clears it);
 * the context stays usable and the next fused call on the workspace clears
 * the barrier's counter.  No fault, trap or hang is involved.
 *   workspace  device, >= 256 bytes, 256-byte aligned (its flag block is used).
 * Returns HS2_OK once launched (asynchronous on `stream`).
 */
int hs2_selftest_grid_barrier(void *workspace, size_t workspace_bytes, void *stream);

/*
 * The same self-test on the static scratch of hs2_full_attn_select_static()
 * in the current CUDA context: afterwards hs2_full_attn_select_static_status()
 * returns HS2_ERR_TIMEOUT once (and clears the flag).  Must not overlap a
 * static call on the GPU.
 */
int hs2_selftest_bounded_wait_static(void *stream);

const char *hs2_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int hs2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HS2_H_ */
