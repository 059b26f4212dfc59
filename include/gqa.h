/*
 * gqa.h -- C ABI of libgqa: Qwen2-style grouped-query causal self-attention with RoPE
 * on one NVIDIA B200 (sm_100a).
 *
 * The operation (page "Qwen2 architecture introduction", aicoding.csdn.net, §4.1.2-§4.1.3;
 * page "Qwen2架构解析：GQA与MoE技术在大模型中的创新应用", intelliparadigm.com, §2.3 and §3.1):
 *   g = h_q / h_kv query heads share each key/value head; query head t (0-based) reads
 *   KV group u = t / g.  Q and K rows at position m are rotated (RoPE) pair by pair,
 *   dimension i with i + d/2, by the angle m * theta^(-2i/d).  Per head,
 *   S = Q' K'^T / sqrt(d), S_ij = -inf for j > i (causal), A = softmax(S), head_t = A V_u.
 *
 * Conventions for every entry point below
 *   - All tensor pointers are DEVICE pointers owned by the caller, bf16 (bfloat16, stored
 *     as 16-bit words), dense row-major with exactly the shapes given, 16-byte aligned.
 *   - Work is enqueued on the stream set by gqa_set_stream() (default: the legacy stream 0)
 *     and runs asynchronously; no call below synchronises the host except gqa_last_error()
 *     and the first call on a device (one-time device query).
 *   - Return value: 0 on success, or one of the negative GQA_ERR_* codes.  A failing call
 *     launches nothing and leaves `out` untouched.  Library code never traps or aborts.
 *   - Not thread-safe: the stream and the workspace are process-global state.  Calls that can
 *     overlap on the GPU (enqueued on different streams without synchronisation between them)
 *     share that workspace and the cached attention schedule and race: keep such calls on one
 *     stream, or synchronise between them.
 */
#ifndef GQA_H_
#define GQA_H_

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define GQA_OK 0
#define GQA_ERR_NULL (-1)      /* a required pointer is NULL                                  */
#define GQA_ERR_DIMS (-2)      /* B, L < 0; h_q, h_kv <= 0; h_q % h_kv != 0; or sizes too large */
#define GQA_ERR_HEAD_DIM (-3)  /* d is not 64 or 128                                          */
#define GQA_ERR_THETA (-4)     /* theta <= 0 or not finite                                    */
#define GQA_ERR_LAUNCH (-5)    /* a CUDA launch or tensor-map encode failed                   */
#define GQA_ERR_ALLOC (-6)     /* the internal workspace could not be allocated               */
#define GQA_ERR_ALIGN (-7)     /* a tensor pointer is not 16-byte aligned                     */
#define GQA_ERR_DEVICE (-8)    /* the current device is not an sm_100 (B200-class) GPU        */
#define GQA_ERR_TOO_LARGE (-9) /* gqa_decode_noalloc: more scratch needed than its fixed buffer */

/* Bits of the device error word returned by gqa_last_error(). */
#define GQA_DEVERR_SEQLEN 1    /* a decode length was <= 0; that sequence's output was zeroed */
#define GQA_DEVERR_TIMEOUT 2   /* a kernel pipeline wait ran past its limit and gave up;     */
                               /* outputs of that call are undefined                          */
#define GQA_DEVERR_PAGE 4      /* gqa_decode_paged: a cache row had no valid block-table entry */
                               /* (page index outside [0, num_pages), or the sequence is longer */
                               /* than max_pages_per_seq pages); that row was read as zeros     */

/*
 * Causal GQA prefill over whole sequences (page "Qwen2 architecture introduction",
 * §4.1.3 steps 3-5).
 *   q   [B, L, h_q,  d]   token-major: the per-head split of the Q projection output
 *   k   [B, L, h_kv, d]   un-rotated keys
 *   v   [B, L, h_kv, d]
 *   out [B, L, h_q,  d]   head_t rows, i.e. the concatenation [head_1 | ... | head_hq]
 * Positions are 0 .. L-1 in every batch row.  d in {64, 128}; h_q % h_kv == 0; any L >= 1
 * (a ragged last tile is handled).  B == 0 or L == 0 is a no-op that returns GQA_OK.
 * Uses an internal device workspace (rotated Q and K, B*(h_q+h_kv)*L*d*2 bytes), grown on
 * demand and kept until gqa_release().  The first call for a new (B, L, h_q, h_kv) also plans
 * the attention kernel's work schedule on the host and copies it to the device (a few KB, kept
 * until the shape changes; see gqa_prefill_schedule): to capture calls into a CUDA graph, make
 * one call of the shape before capturing.
 * theta is the RoPE base (Qwen2: 1e6).
 */
GQA_API int gqa_prefill(const void* q, const void* k, const void* v, void* out,
                int B, int L, int h_q, int h_kv, int d, float theta);

/*
 * One decode step: one new query token per sequence against a packed KV cache
 * (page "Qwen2 architecture introduction", §4.1.3 closing paragraph: only the h_kv groups
 * are cached; page "从 Qwen 1 到 Qwen 2", nxmr.cn, §2.4).
 *   q       [B, h_q, d]
 *   kcache  [sum(seqlens), h_kv, d]   un-rotated keys, sequences concatenated in b order:
 *   vcache  [sum(seqlens), h_kv, d]   row j of sequence b is packed row off_b + j,
 *                                     off_b = seqlens[0] + ... + seqlens[b-1]
 *   seqlens [B] int32, DEVICE memory; each >= 1
 *   out     [B, h_q, d]
 * The query of sequence b sits at position seqlens[b] and attends to all seqlens[b] cached
 * rows (positions 0 .. seqlens[b]-1).  A length <= 0 is not an API error (lengths live on
 * the device): that sequence's output is zeroed and GQA_DEVERR_SEQLEN is raised in the device
 * error word.  B == 0 is a no-op.  Uses an internal workspace (packed offsets and split
 * partials, a few MB), grown on demand and kept until gqa_release().
 */
GQA_API int gqa_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens,
               void* out, int B, int h_q, int h_kv, int d, float theta);

/*
 * Measurement support.  With both events non-NULL (cudaEvent_t handles passed as void*, created
 * by the caller), every later gqa_prefill / gqa_decode call records `start` on the current stream
 * right before its main kernel and `stop` right after it: the attention kernel of the prefill,
 * the split kernel of the decode.  The caller owns the events.  NULL, NULL turns this off.
 */
GQA_API int gqa_set_timing_events(void* start_event, void* stop_event);

/*
 * gqa_decode_noalloc -- the same decode step as gqa_decode (same arguments, layouts, results and
 * error codes), for callers that cannot let the library allocate device memory.  No counterpart in
 * the paper: this is a library-level variant.
 *
 * Who needs it: a caller that owns all device memory itself (e.g. a serving process that reserves
 * nearly all of HBM for its KV cache and weights up front, where a cudaMalloc from inside a library
 * would fail or fragment that reservation), or a caller on a latency-critical path that cannot pay
 * for cudaMalloc / cudaFree, which may synchronise the whole device.  This entry point calls no
 * cudaMalloc, cudaFree or other allocating routine.  Its scratch (packed row offsets and split
 * partials) is a fixed 16 MiB array in the library's device memory, which every GPU that loads the
 * library holds until the process exits.
 *
 * Limit: the scratch needed is 8*(B+1) bytes rounded up to a multiple of 256, plus
 * (P + B) * h_kv * ceil(g/8) * (16 + 8*d) * 4 bytes, where P = 4 * ceil(3*SMs / (h_kv*ceil(g/8)))
 * (3 split CTAs of 4 warps per SM; P = 444 for h_kv = 4, g = 7 on a 148-SM B200, so the Qwen2-7B
 * shape fits up to B = 563).  The total must not exceed 16 MiB (16777216 bytes); larger problems
 * return GQA_ERR_TOO_LARGE and launch nothing.
 *
 * The first call on a device looks up the device address of the fixed array (with that device
 * current); make that first call before any stream capture.  All calls on a device share the one
 * array and each leaves its contents behind; nothing in it has to start at zero.  Calls whose work
 * overlaps on the GPU (different streams, or different host threads) race on the array: serialise
 * them on one stream.
 */
GQA_API int gqa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                               void* out, int B, int h_q, int h_kv, int d, float theta);

/*
 * gqa_decode_paged -- the decode step of gqa_decode over a paged KV cache (page "从 Qwen 1 到 Qwen 2",
 * nxmr.cn, §2.4: serving engines such as vLLM keep the cache of each KV head in fixed-size blocks,
 * PagedAttention).  Same query, positions, softmax and output as gqa_decode; only where cache rows live
 * differs.
 *   kpages, vpages [num_pages, page_size, h_kv, d]   un-rotated keys / values; page P slot s holds one
 *                                                    cache row (all h_kv heads of one position)
 *   block_table    [B, max_pages_per_seq] int32, DEVICE memory: row j (position j, 0-based) of sequence b
 *                  lives in page block_table[b][j / page_size], slot j % page_size.  Entries for pages past
 *                  the end of a sequence are not read.  Pages may be shared between sequences.
 *   seqlens [B] int32 DEVICE memory, q [B, h_q, d], out [B, h_q, d], d and theta as for gqa_decode.
 * page_size >= 1 (any value; 16 or a multiple of 16 keeps whole blocks of 16 rows in one page),
 * num_pages >= 1, max_pages_per_seq >= 1, else GQA_ERR_DIMS.  A table entry outside [0, num_pages), or a
 * sequence longer than max_pages_per_seq * page_size, is not an API error (the table lives on the
 * device): the rows concerned are read as zeros, nothing outside kpages / vpages is accessed, and
 * GQA_DEVERR_PAGE is raised in the device error word.  Workspace and stream as for gqa_decode.
 */
GQA_API int gqa_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                             const int* seqlens, void* out, int B, int h_q, int h_kv, int d, int page_size,
                             int num_pages, int max_pages_per_seq, float theta);

/*
 * gqa_qkv_rope -- the step before the attention, fused (page "Qwen2 architecture introduction",
 * aicoding.csdn.net, §4.1.3 steps 1-3): the Q, K, V projections with their bias, the split into h_q query
 * heads and h_kv key/value heads, and RoPE on Q and K; it also writes the KV-cache rows of the sequences.
 *   x      [B, L, d_model]                 hidden states (after RMSNorm), bf16
 *   w_qkv  [(h_q + 2 h_kv) d, d_model]     rows 0 .. h_q d - 1 are W_Q^T, then W_K^T, then W_V^T (the
 *                                          nn.Linear weight layout: output feature major), bf16
 *   b_qkv  [(h_q + 2 h_kv) d]              the matching bias, bf16, or NULL for none
 * Outputs (bf16, caller-owned): with Y = x w_qkv^T + b_qkv split into heads, at positions 0 .. L-1,
 *   qr [B, h_q, L, d]   rotated Q, head-major      kr [B, h_kv, L, d]   rotated K, head-major
 *   k  [B, L, h_kv, d]  un-rotated K, token-major  v  [B, L, h_kv, d]   V, token-major
 *   (k holds the rotated K instead while gqa_set_decode_cache_rotated(1) is in effect)
 * k and v are exactly the packed cache rows of gqa_decode for B sequences of L rows stored back to back,
 * so pointing them into a cache appends the sequences; qr, kr and v are the inputs of
 * gqa_prefill_rotated.  Each output element is the fp32 accumulation rounded to bf16 once.
 * d in {64, 128}; d_model a positive multiple of 8; all pointers 16-byte aligned.  B == 0 or L == 0 is a
 * no-op.  Uses an internal device table of cos / sin for positions 0 .. L-1 (L * d/2 * 8 bytes), rebuilt
 * when L, d or theta change and kept until gqa_release().
 */
GQA_API int gqa_qkv_rope(const void* x, const void* w_qkv, const void* b_qkv, void* qr, void* kr, void* k, void* v,
                         int B, int L, int d_model, int h_q, int h_kv, int d, float theta);

/*
 * gqa_qkv_append -- one decode step's projection with its cache append (page "Qwen2 architecture
 * introduction", aicoding.csdn.net, §4.1.3 steps 1-2 and closing paragraph: each decode step projects the
 * new token and appends its K and V to the cache of the h_kv groups; page "从 Qwen 1 到 Qwen 2", nxmr.cn,
 * §2.4: that cache kept in pages, as gqa_decode_paged reads it).
 *   x            [B, d_model]  the new token of each of B sequences (hidden states after RMSNorm), bf16
 *   w_qkv, b_qkv as for gqa_qkv_rope (b_qkv may be NULL)
 *   seqlens      [B] int32, DEVICE memory: each sequence's cache length before the append, i.e. the
 *                position p_b of its new token
 *   q            [B, h_q, d]   out: the new tokens' queries, un-rotated (the decode entry points rotate the
 *                query at its position)
 *   kpages, vpages [num_pages, page_size, h_kv, d]  the paged cache of gqa_decode_paged: the token's K
 *                (un-rotated, like every cache row; rotated at p_b when the caches keep keys after RoPE,
 *                see gqa_set_decode_cache_rotated) and V are written to slot p_b % page_size of page
 *                block_table[b][p_b / page_size]; nothing else in the pages is touched
 *   block_table  [B, max_pages_per_seq] int32, DEVICE memory
 *   theta        the RoPE base of that key rotation (used only when the caches keep rotated keys; must be
 *                finite and > 0 in any case, else GQA_ERR_THETA)
 * Each written element is the fp32 accumulation (plus the bias) rounded once to bf16.  A decode loop is
 * then: gqa_qkv_append, then gqa_decode_paged with seqlens[b] + 1 and gqa_set_decode_self_in_cache(1) (the
 * new token attends to itself and to every earlier position), then grow seqlens.  A position outside the
 * table (p_b < 0, or p_b / page_size >= max_pages_per_seq) or a table entry outside [0, num_pages) is not
 * an API error (both live on the device): that token's K and V are not written and GQA_DEVERR_PAGE is
 * raised; its q is still written.  Sizes as for gqa_qkv_rope and gqa_decode_paged; B == 0 is a no-op.
 */
GQA_API int gqa_qkv_append(const void* x, const void* w_qkv, const void* b_qkv, const int* seqlens, void* q,
                           void* kpages, void* vpages, const int* block_table, int B, int d_model, int h_q,
                           int h_kv, int d, int page_size, int num_pages, int max_pages_per_seq, float theta);

/*
 * gqa_set_decode_self_in_cache -- where the query of every later gqa_decode, gqa_decode_paged and
 * gqa_decode_noalloc call sits.  0 (the default): at position seqlens[b], attending to the seqlens[b]
 * cached rows before it, which do not include the query's own row.  1: the cache already holds the query's
 * own K and V as its last row (appended by gqa_qkv_append, the order of page "Qwen2 architecture
 * introduction", §4.1.3 closing paragraph), so the query sits at position seqlens[b] - 1 and attends to all
 * seqlens[b] rows, itself included.  Process-global, like the stream.  Returns GQA_ERR_DIMS for other values.
 */
GQA_API int gqa_set_decode_self_in_cache(int on);

/*
 * gqa_set_decode_cache_rotated -- what the K cache holds for every later gqa_decode, gqa_decode_paged,
 * gqa_decode_noalloc and gqa_qkv_append call, and what gqa_qkv_rope writes to its k output.  0 (the
 * default): raw keys, as projected; the decode rotates each cached key at its row index on load (page
 * "Qwen2 architecture introduction", §4.1.3: RoPE acts on Q and K before the dot product).  1: keys kept
 * after RoPE, each already rotated at its own position (with the YaRN temperature when scaling is on), as
 * a serving cache keeps them; the decode uses them as loaded and rotates only the query, gqa_qkv_append
 * writes the new key rotated at its position, and gqa_qkv_rope's k output holds the rotated keys
 * (token-major; kr is unchanged).  The scores are the same either way; the rotated cache saves the decode
 * the per-key rotation.  Process-global, like the stream.  Returns GQA_ERR_DIMS for other values.
 */
GQA_API int gqa_set_decode_cache_rotated(int on);

/*
 * gqa_prefill_rotated -- the causal attention of gqa_prefill on inputs that are already rotated (page
 * "Qwen2 architecture introduction", §4.1.3 steps 4-5): qr [B, h_q, L, d] and kr [B, h_kv, L, d]
 * head-major as gqa_qkv_rope writes them, v [B, L, h_kv, d], out [B, L, h_q, d].  No RoPE and no
 * workspace: the prep pass of gqa_prefill is skipped.  Same checks and conventions as gqa_prefill.
 */
GQA_API int gqa_prefill_rotated(const void* qr, const void* kr, const void* v, void* out, int B, int L, int h_q,
                                int h_kv, int d);

/*
 * gqa_out_proj -- the step after the attention (page "Qwen2 architecture introduction", §4.1.3 steps 5-6):
 * the concatenated heads times W_O, plus the residual:  out = attn w_o^T + residual.
 *   attn     [T, d_in]       the attention output viewed as rows: gqa_prefill's out [B, L, h_q, d] is
 *                            already this Concat with T = B*L, d_in = h_q d
 *   w_o      [d_model, d_in] rows of W_O^T (the nn.Linear weight layout), bf16
 *   residual [T, d_model]    the sub-layer input X_in, or NULL for none
 *   out      [T, d_model]    may be the same buffer as residual (updated in place)
 * Each element is the fp32 accumulation (plus the residual in fp32) rounded once to bf16.  d_in a positive
 * multiple of 8, d_model a positive multiple of 128, pointers 16-byte aligned; T == 0 is a no-op.
 */
GQA_API int gqa_out_proj(const void* attn, const void* w_o, const void* residual, void* out, int T, int d_in,
                         int d_model);

/*
 * gqa_set_rope_scaling -- YaRN scaling of RoPE for every later gqa_prefill, gqa_decode, gqa_decode_paged,
 * gqa_decode_noalloc and gqa_qkv_rope call, for contexts beyond the trained window (page "Qwen-2
 * explained", yudonglee.me, §6.2: frequencies f_i / s * alpha_i with a per-pair ramp alpha_i; page "Qwen2
 * architecture introduction", aicoding.csdn.net, §5.3: the attention logits are rescaled).  The pages give
 * neither the ramp's bounds nor the rescaling; both follow the published YaRN method: alpha_i = 1 +
 * gamma_i (s - 1) with gamma_i = clamp((r_i - 1) / 31, 0, 1), r_i = original_max_position * f_i / (2 pi),
 * and the logits multiplied by (0.1 ln s + 1)^2.
 *   factor                 s >= 1; 1 turns scaling off (the default)
 *   original_max_position  the trained window (Qwen2: 32768); must be > 0 when factor > 1
 * The page (aicoding.csdn.net, §5.5) notes the scaled model behaves as the plain one within the trained
 * window: enabling scaling only for contexts longer than it is left to the caller.  gqa_prefill_rotated
 * takes Q' and K' as given (gqa_qkv_rope folds the temperature into them).  Process-global, like the
 * stream; returns GQA_ERR_DIMS for invalid values (the setting is then unchanged).
 */
GQA_API int gqa_set_rope_scaling(float factor, int original_max_position);

/* Stream for subsequent calls (a cudaStream_t passed as void*; NULL = legacy stream). */
GQA_API int gqa_set_stream(void* cuda_stream);

/*
 * Synchronises the current stream, then returns and clears the device error word of the
 * current device (a combination of GQA_DEVERR_* bits; 0 if clean), or GQA_ERR_LAUNCH if
 * the stream reports a CUDA error.
 */
GQA_API int gqa_last_error(void);

/*
 * gqa_prefill_schedule -- how gqa_prefill and gqa_prefill_rotated deal their attention work out over `grid`
 * persistent CTAs (one per SM: pass the SM count), computed on the host exactly as the library does it;
 * no device is needed.  For inspection and tests.
 * The work items are pairs of 128-row query tiles of one (batch row, KV group): item w covers the tiles
 * 2(w / (B*h_kv)) and 2(w / (B*h_kv)) + 1 of the group b*h_kv + u = w mod (B*h_kv), whose tiles are listed
 * by query tile descending, then head ascending (causal masking: tile index i needs L/128 - i/g key tiles).
 * With more items than CTAs, each CTA takes its items in the listed order.  Where there are few items per
 * CTA they are packed by best fit decreasing on (key tiles + a fixed per-item cost), for balance.  Where a
 * plain round-robin order (every other round reversed) is already within 2 % of that packing, it is used
 * as it is if the K' and V of all (b, u) planes fit in 48 MB (at d = 128), and otherwise (*grouped = 1) the
 * items are dealt for L2 reuse: the planes a group at a time (as many as keep 16 MB of K' and V, at least
 * one), each group's items heaviest first to the least loaded CTA.
 *   starts  [min(grid, items) + 1] CTA c's items are items[starts[c] .. starts[c+1])   (caller-owned)
 *   items   [items]                                                                   (caller-owned)
 *   capacity  the room in items; the arrays are written only when it suffices (and both are non-null)
 * Returns the number of items (>= 0), or GQA_ERR_DIMS for non-positive sizes, h_q % h_kv != 0 or sizes
 * gqa_prefill rejects.
 */
GQA_API int gqa_prefill_schedule(int B, int L, int h_q, int h_kv, int grid, int* starts, int* items, int capacity,
                                 int* grouped);

/* Frees the internal workspaces (and the cos / sin table) of every device this process used (synchronises each). */
GQA_API void gqa_release(void);

/* Static, human-readable text for a GQA_ERR_* code. */
GQA_API const char* gqa_strerror(int code);

/* ABI version of this header (incremented on incompatible changes). */
GQA_API int gqa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H_ */
