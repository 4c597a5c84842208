/*
 * segpaged.h -- C ABI of the SegPagedAttention library for NVIDIA B200 (sm_100a).
 *
 * SegPagedAttention stores the KV cache as pages keyed by (layer, head, segment) instead of a
 * dense [B, H, L, D] tensor. A global head keeps its whole context; a local head physically keeps
 * only its sink tokens and its recent window. One mask-free, variable-length attention kernel runs
 * every head over exactly its own ragged KV.
 *   Sources: "小红书把 KV Cache 按「头」拆了" (zhichai.net), 事件内容 item 3 "SegPagedAttention 存储";
 *   "RedKnot – 小红书研发并开源的长上下文大模型推理引擎" (shshi.cn), 技术原理 1 "SegPagedAttention存储架构";
 *   "为什么长上下文推理这么慢？RedKnot…" (bjdmk.com.cn), 二 "三大核心机制" item 3;
 *   "RedKnot - Xiaohongshuが開発した…" (aiboss88.com), 技術原則, item on paged storage removing the
 *   attn_mask kernel penalty.
 *
 * The calls follow the four adapters the last page names (使い方): BUILDSTATE -> segpaged_build,
 * SELECTVISIBLESTATE -> segpaged_prefill_plan, EXECUTE -> segpaged_attn_prefill; PROFILE (the
 * offline head classification) happens outside this library and reaches it as the class map.
 *
 * Conventions shared by every call
 *  - Visibility. Query position i of a sequence sees key j iff j <= i and (the KV head is global, or
 *    j < sink, or j > i - window). Queries are the Lq tail positions L-Lq .. L-1 of a sequence of
 *    context length L. Query head h reads KV head h / G, G = num_q_heads / num_kv_heads.
 *  - Stored pages. Logical page n of a (sequence, KV head) holds tokens [n*P, n*P+P). A global head
 *    stores pages 0 .. ceil(L/P)-1. A local head stores the pages holding a token < min(sink, L) and
 *    the pages holding a token >= max(L - Lq - window + 1, 0). The page table of a (sequence, KV
 *    head) lists the physical page of each stored logical page in ascending logical order
 *    (sink pages first, then window pages). Physical ids may be any permutation.
 *  - Layouts (row-major, bf16 unless stated): dense K/V [sum L_b, Hkv, D]; Q and O
 *    [sum Lq_b, Hq, D]; LSE float32 [Hq, sum Lq_b] (natural log); pools [num_pages, P, D].
 *  - Page-table arrays are flattened over (sequence b, KV head k) in b-major order: entries of head
 *    (b, k) are page_table[offs[b*Hkv + k] .. offs[b*Hkv + k + 1]).
 *  - Ownership. Every pointer is owned by the caller; the library keeps none after a call returns
 *    and allocates no device memory. "dev" pointers are device memory, "host" pointers host memory.
 *  - Streams. Device work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream) and is asynchronous to the host.
 *  - Errors. A call returns 0 (or a count) on success and a negative SEGPAGED_ERR_* code otherwise;
 *    on a host-detected error nothing is enqueued. Device-side checks (a page id outside
 *    [0, num_pages), a page table whose length disagrees with the storage rule, a pipeline wait that
 *    timed out) OR a SEGPAGED_STATUS_* bit into the optional device status word and keep all
 *    memory accesses in bounds; the caller reads the word after synchronising.
 *  - Supported shapes: head_dim in {64, 128}; page_size in {16, 32, 64, 128}; G a power of two
 *    <= 128; base pointers of q, pools and o 16-byte aligned.
 */
#ifndef SEGPAGED_H
#define SEGPAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SEGPAGED_OK 0
#define SEGPAGED_ERR_NULL (-1)      /* a required pointer is NULL */
#define SEGPAGED_ERR_DIMS (-2)      /* unsupported or inconsistent dims */
#define SEGPAGED_ERR_CLASS (-3)     /* head class out of range (sink < 0, window < 1 for a local head) */
#define SEGPAGED_ERR_SEQ (-4)       /* negative length, or Lq > L */
#define SEGPAGED_ERR_PAGES (-5)     /* page-table offsets disagree with the storage rule */
#define SEGPAGED_ERR_CAPACITY (-6)  /* output array too small */
#define SEGPAGED_ERR_CUDA (-7)      /* a CUDA runtime/driver call failed */
#define SEGPAGED_ERR_ALIGN (-8)     /* a base pointer is not 16-byte aligned */
#define SEGPAGED_ERR_UNSUPPORTED (-9) /* the plan splits units, which this entry point does not accept */

#define SEGPAGED_STATUS_PAGE_ID 1   /* a page id was outside [0, num_pages); it was clamped */
#define SEGPAGED_STATUS_TABLE 2     /* a head's page-table length disagreed with the storage rule */
#define SEGPAGED_STATUS_TIMEOUT 4   /* a pipeline wait gave up; outputs of this call are undefined */
#define SEGPAGED_STATUS_UNIT 8      /* a plan record did not fit the page table or the call: entries past the
                                       page table, or a plan that disagrees with its info or entry point */

typedef struct {
  int32_t num_seqs;      /* B */
  int32_t num_q_heads;   /* Hq */
  int32_t num_kv_heads;  /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;      /* D */
  int32_t page_size;     /* P, tokens per page */
  int32_t num_pages;     /* physical pages in each of k_pool and v_pool */
} segpaged_dims;

/* Class of one (sequence, KV head) of one layer: the offline head classification. */
typedef struct {
  int32_t is_global;  /* 1: full causal context; 0: local */
  int32_t sink;       /* S >= 0, local heads only */
  int32_t window;     /* W >= 1, local heads only */
} segpaged_head_class;

/* One record of a prefill plan: a work unit -- a (sequence, KV head) and up to 2 x 128/G query
 * positions, with its visible page ranges and the KV tiles it runs -- or a combine record that merges
 * the chunks of a split unit. Produced by segpaged_prefill_plan; the fields are private. 128 bytes. */
typedef struct {
  int32_t v[32];
} segpaged_unit;

/* Shape of a plan: records [0, num_units) are work units, records [num_units, num_units + num_groups)
 * combine records; num_partials partial-result slots live in the workspace; num_half_units of the units
 * have rows in one query tile only. num_half_units only picks a kernel variant (> 0: each such unit's KV
 * tiles alternate between both softmax warpgroups, which merge their two partial results at the end;
 * == num_units: the unused second query buffer also serves as one more K/V slot); results are correct
 * for any value below num_units, but the variants round differently. combine_row_blocks sizes the
 * combine launch: the most blocks of 32 rows one combine record needs, 0 for "unknown" (8, a whole
 * record). A value below what the plan needs leaves rows unmerged and sets SEGPAGED_STATUS_UNIT.
 * The last six fields record the call the plan was made for: its records address query rows
 * [0, total_q), query heads [0, num_q_heads) and page-table entries [0, page_table_len) (the planner's
 * page_table_offs[B*Hkv]). The prefill entry points return SEGPAGED_ERR_DIMS before any launch when the
 * call's total_q, num_q_heads, num_kv_heads, head_dim or page_size differ from them or its page table is
 * shorter, and the kernels skip (and report with SEGPAGED_STATUS_UNIT) any output row, head or partial
 * slot a record names outside the call's arrays. */
typedef struct {
  int64_t num_units;
  int64_t num_groups;
  int64_t num_partials;
  int64_t num_half_units;
  int64_t combine_row_blocks;
  int64_t total_q;
  int64_t page_table_len;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
} segpaged_plan_info;

/* Text for an error code (static storage). */
const char* segpaged_error_string(int code);

/*
 * Physical KV footprint of a layer (host only, no device work).
 *   ctx_len[B], q_len[B] (host): L_b and Lq_b.  cls[B*Hkv] (host).
 *   pages_per_head[B*Hkv] (host, nullable): stored page count of each (b, k).
 *   dense_bytes (host, nullable): K+V bytes if every KV head kept all ceil(L_b/P) pages.
 * Returns the stored K+V bytes (num stored pages * P * D * 2 tensors * 2 bytes), or an error code.
 * Source: the physically sparse access of SegPagedAttention, which cuts the KV bytes moved
 * (shshi.cn, 技术原理 1, "物理级稀疏访问").
 */
int64_t segpaged_pages_bytes(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                             const segpaged_head_class* cls, int64_t* dense_bytes, int32_t* pages_per_head);

/*
 * RoPE re-alignment table (host only). out[b][d][0..1] = (cos, sin) of deltas[b] * theta^(-2d/D),
 * d in [0, D/2), evaluated in double and rounded to float. out is host [num_seqs, D/2, 2].
 * Source: rotating offline-computed keys from their original to their actual position
 * (shshi.cn, 技术原理 2 "位置无关缓存复用", item "RoPE位置对齐").
 */
int segpaged_rope_cos_sin(double theta, const int32_t* deltas, int32_t num_seqs, int32_t head_dim, float* out);

/*
 * BUILDSTATE: scatter a layer's dense K/V into the page pools (one kernel launch).
 *   k_dense, v_dense (dev): [sum L_b, Hkv, D] bf16.   cu_seqlens_k (dev) [B+1]: token offsets.
 *   q_len (dev) [B]: Lq_b, which fixes the window pages a local head stores.  cls (dev) [B*Hkv].
 *   page_table (dev, int32) and page_table_offs (dev, int32 [B*Hkv+1]) as described above.
 *   rope_cos_sin (dev, nullable) [B, D/2, 2] float from segpaged_rope_cos_sin: when set, every
 *     stored key is rotated (rotate-half pairs (d, d+D/2)): y1 = x1*c - x2*s, y2 = x2*c + x1*s,
 *     each product and sum rounded to float, then rounded to bf16 (nearest even). V is copied as is.
 *   k_pool, v_pool (dev) [num_pages, P, D] bf16: each stored page receives its P rows; rows past
 *     L_b are written as zero. Pages not named by any table are not touched.
 *   status (dev, nullable): see SEGPAGED_STATUS_*.
 * Sources: the BUILDSTATE adapter, which precomputes fragment KV and stores it page by page per head
 *   into the global/local pools (aiboss88.com, 使い方, second item); the RoPE re-alignment
 *   (shshi.cn, 技术原理 2, item "RoPE位置对齐").
 */
int segpaged_build(const segpaged_dims* dims, const void* k_dense, const void* v_dense,
                   const int32_t* cu_seqlens_k, const int32_t* q_len, const segpaged_head_class* cls,
                   const int32_t* page_table, const int32_t* page_table_offs, const float* rope_cos_sin,
                   void* k_pool, void* v_pool, int32_t* status, void* stream);

/*
 * SELECTVISIBLESTATE: plan the prefill work (host only).
 * Splits every (sequence, KV head) into units of 2 x 128/G positions x G query heads (two 128-row
 * tensor-core tiles sharing each K/V tile), records for each the page ranges its queries can see (the
 * sink pages and the window pages, in page-table index space) and orders them longest-first by cost
 * bucket, keeping units of one head together inside a bucket.
 * With split_ctas > 0 (the number of CTAs that run concurrently, e.g. the SM count) and a unit longer
 * than a CTA's fair share of the work -- short query ranges, decode-like tiles -- long units are cut
 * into chunks of at least 8 KV tiles; each chunk writes a partial result and a combine record merges
 * them in chunk order (deterministic). split_ctas = 0 never splits.
 *   ctx_len, q_len (host) [B]; cls (host) [B*Hkv]; page_table_offs (host) [B*Hkv+1] (the same
 *   offsets later given to the device), checked against the storage rule.
 *   units (host, nullable) [capacity]; info (host, nullable) receives the plan's shape.
 * Returns the number of records (work units + combine records; also when units is NULL, to size the
 * array), or an error code. The caller copies the records to device memory for segpaged_attn_prefill;
 * a plan stays valid for any call with the same lengths, classes and offsets.
 * Source: the SELECTVISIBLESTATE adapter, which picks the local-head KV to reuse and the global-head
 *   ranges to compute (aiboss88.com, 使い方, third item).
 */
int64_t segpaged_prefill_plan(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                              const segpaged_head_class* cls, const int32_t* page_table_offs, int32_t split_ctas,
                              segpaged_unit* units, int64_t capacity, segpaged_plan_info* info);

/* Plans the fused append-and-attend call (segpaged_attn_prefill_append); same inputs and outputs as
 * segpaged_prefill_plan. Each unit reads the keys before its sequence's query range from the pool and the
 * keys from the query range on from the new K/V. Give the plan to segpaged_attn_prefill_append only. */
int64_t segpaged_prefill_plan_append(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                                     const segpaged_head_class* cls, const int32_t* page_table_offs,
                                     int32_t split_ctas, segpaged_unit* units, int64_t capacity,
                                     segpaged_plan_info* info);

/* Device scratch bytes segpaged_attn_prefill needs for a plan: the work counter and, for split plans,
 * the partial results (256 x D + 256 floats per partial slot). */
size_t segpaged_prefill_workspace_bytes(const segpaged_dims* dims, const segpaged_plan_info* info);

/*
 * EXECUTE: causal attention of every query head over its own ragged paged KV (one persistent
 * kernel launch, preceded by a 4-byte memset of the workspace's work counter when the plan has more
 * units than the GPU has SMs; for split plans followed by one combine launch).
 *   q (dev) [total_q, Hq, D] bf16.  k_pool, v_pool (dev) [num_pages, P, D] bf16.
 *   page_table (dev, int32) [page_table_len].
 *   plan (dev) [info->num_units + info->num_groups] records from segpaged_prefill_plan; info (host).
 *     The plan must come from the same dims, lengths, classes and offsets as this call, and info must be
 *     the one the planner returned with it. A call whose total_q, heads, head_dim, page_size or page
 *     table length disagree with info returns SEGPAGED_ERR_DIMS before any launch; a record that still
 *     names a row, head, page-table entry or partial slot outside the call's arrays (records from another
 *     plan than info's) is skipped and sets SEGPAGED_STATUS_UNIT.
 *   softmax_scale: logits are scale * q.k (1/sqrt(D) in the usual case).
 *   o (dev) [total_q, Hq, D] bf16: O = softmax(logits over the visible keys) . V.
 *   lse (dev) [Hq, total_q] float: natural-log sum of exp(logits) over the visible keys.
 *   workspace (dev) >= segpaged_prefill_workspace_bytes(dims, info), 16-byte aligned.
 *   status (dev, nullable): see SEGPAGED_STATUS_*.
 * Every stored page slot must hold finite values (segpaged_build writes zeros past the context end).
 * Sources: one fused variable-length attention kernel that keeps every head on the fast path and
 *   builds no attention mask (zhichai.net, 事件内容 item 3); global heads read all context pages and
 *   local heads only their sink and recent-window pages, run by a mask-free varlen kernel
 *   (bjdmk.com.cn, 二 item 3); the EXECUTE adapter (aiboss88.com, 使い方, fourth item).
 */
int segpaged_attn_prefill(const segpaged_dims* dims, const void* q, int32_t total_q,
                          const void* k_pool, const void* v_pool, const int32_t* page_table,
                          int64_t page_table_len, const segpaged_unit* plan, const segpaged_plan_info* info,
                          float softmax_scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                          int32_t* status, void* stream);

/*
 * EXECUTE fused with the append of the new tokens' keys and values into the pool (the online KV cache the
 * recompute writes: aiboss88.com, 使い方, fourth item "EXECUTE" writes global-head recompute into the online
 * KV cache), in one launch. Arguments as segpaged_attn_prefill, plus
 *   k_new, v_new (dev) [total_q, Hkv, D] bf16, 16-byte aligned: the keys and values of the query rows
 *     (position L - Lq + r of sequence b for row cu_q[b] + r), as the model computed them;
 *   plan from segpaged_prefill_plan_append.
 * Effects: every pool row of a query position of every (sequence, KV head) is overwritten with its new key
 * and value (each exactly once), and O / LSE are the attention over the pool's rows before the query
 * range and the new rows from it on -- the same result as segpaged_build of the full K/V followed by
 * segpaged_attn_prefill, up to floating-point order. Pool rows of the query range are never read, so they
 * may hold anything finite beforehand; the pages they live in must be in the page table (the storage rule
 * keeps every page with a query position).
 */
int segpaged_attn_prefill_append(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_new,
                                 const void* v_new, void* k_pool, void* v_pool, const int32_t* page_table,
                                 int64_t page_table_len, const segpaged_unit* plan, const segpaged_plan_info* info,
                                 float softmax_scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                                 int32_t* status, void* stream);

/*
 * The same per-fragment RoPE re-alignment as segpaged_attn_prefill_rope, done once per request instead of
 * at every K tile load: every stored page of every (sequence, KV head) of one layer is copied from k_pool to
 * k_pool_out at the same physical id, with the rows whose token falls in a fragment rotated (same rule,
 * same rounding). segpaged_attn_prefill run with k_pool_out as its K pool then gives bit-identical results
 * to segpaged_attn_prefill_rope on k_pool. One pass over the layer's K pages (read and write, HBM-bound)
 * instead of one rotation per unit that loads a tile; it needs a second K pool (k_pool_out, dev, as large
 * as k_pool; ids outside the layer's tables are left untouched).
 *   cu_seqlens_k, q_len, cls, page_table, page_table_offs (dev): as for segpaged_build.
 *   frag_offs, frag_start, frag_cos_sin (dev): as for segpaged_attn_prefill_rope.
 * Returns SEGPAGED_ERR_DIMS if k_pool_out == k_pool.
 */
int segpaged_rope_realign(const segpaged_dims* dims, const int32_t* cu_seqlens_k, const int32_t* q_len,
                          const segpaged_head_class* cls, const int32_t* page_table, const int32_t* page_table_offs,
                          const int32_t* frag_offs, const int32_t* frag_start, const float* frag_cos_sin,
                          const void* k_pool, void* k_pool_out, int32_t* status, void* stream);

/*
 * EXECUTE with the RoPE re-alignment applied at gather time instead of at build time, so a sequence can
 * hold many reused fragments whose keys were computed at other offsets (shshi.cn, 技术原理 2
 * "位置无关缓存复用", item "RoPE位置对齐"). The pools hold the keys as computed offline; each K tile is
 * rotated in shared memory after it lands and before the logits are formed. Arguments as
 * segpaged_attn_prefill, plus (all dev):
 *   frag_offs (int32) [B+1]: sequence b owns fragments [frag_offs[b], frag_offs[b+1]);
 *   frag_start (int32): token position where each fragment starts, ascending within a sequence;
 *   frag_cos_sin (float, 16-byte aligned) [num_fragments][D/2][2]: the fragment's table for its shift
 *     delta = actual - original position, as segpaged_rope_cos_sin computes it.
 * A key token is rotated with the table of the last fragment of its sequence that starts at or before it;
 * tokens before the first fragment keep their keys. The rotation is the build's (same rounding), so one
 * fragment per sequence starting at 0 gives bit-identical results to segpaged_build with that table
 * followed by segpaged_attn_prefill. V is never rotated.
 */
int segpaged_attn_prefill_rope(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool,
                               const void* v_pool, const int32_t* page_table, int64_t page_table_len,
                               const segpaged_unit* plan, const segpaged_plan_info* info, float softmax_scale,
                               const int32_t* frag_offs, const int32_t* frag_start, const float* frag_cos_sin,
                               void* o, float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                               void* stream);

/*
 * segpaged_attn_prefill without caller-provided device scratch. The paper has no counterpart: this
 * entry point exists for callers that cannot allocate device memory when they run prefill (for
 * example code inside a framework's own memory pool, or a runtime that forbids allocation on its
 * request path), so they cannot provide the unit list and workspace segpaged_attn_prefill needs.
 * It computes the same result from the same arguments, except:
 *   units_host (host) [num_units] straight from segpaged_prefill_plan called with split_ctas = 0 (a
 *     plan with split units returns SEGPAGED_ERR_UNSUPPORTED); it is copied on `stream` into a
 *     library-owned device array, so keep it unchanged until the stream has passed this call
 *     (a pageable buffer is staged before the call returns). Every unit is checked on the host first:
 *     one whose query rows, KV head or page-table entries fall outside this call's total_q, dims or
 *     page_table_len returns SEGPAGED_ERR_DIMS before anything is enqueued;
 *   no workspace arguments.
 * The library-owned array is a static device array of 2 MiB that every GPU loading the library keeps
 * until the process exits; it holds at most 16384 units (more return SEGPAGED_ERR_CAPACITY). The
 * first call on a device looks up the array's device address; make that first call before any
 * stream capture. Every call on a device shares the array and it keeps the last call's contents (the
 * work counter is cleared by every call that reads it): calls whose work overlaps on the GPU race, so serialise
 * them (one stream, or events). Allocates no memory.
 */
int segpaged_attn_prefill_noalloc(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool,
                                  const void* v_pool, const int32_t* page_table, int64_t page_table_len,
                                  const segpaged_unit* units_host, int64_t num_units, float softmax_scale, void* o,
                                  float* lse, int32_t* status, void* stream);

/* ------------------------------------------------------------------------------------------------
 * Token importance for sparse FFN.
 *
 * The pages run the dense FFN only on the top-k tokens by attention score and send the other tokens
 * down the residual identity path, choosing them from the attention signal of the prefill
 * ("RedKnot – 小红书研发并开源的长上下文大模型推理引擎" (shshi.cn), 技术原理 3 "稀疏FFN动态调度";
 * "为什么长上下文推理这么慢？RedKnot…" (bjdmk.com.cn), 二 "三大核心机制" item 2 "稀疏 FFN 与自适应专家
 * Top-K"; zhichai.net, 事件内容 item 2 "稀疏 FFN"). They define neither the score nor the tie rule. The
 * reading taken here: the score of a token of the query range is the attention mass it receives in
 * this prefill,
 *   mass[r] = sum over query heads h and query positions i of exp(s_hij - LSE_hi) for j in V_h(i),
 * where j is the position of query row r (its own key), s the scaled logits of the prefill and LSE
 * its row log-sum-exp. The FFN itself (model weights) is not part of this library.
 * ------------------------------------------------------------------------------------------------ */

/* One work item of a mass plan: a (sequence, KV head, 128-key tile of the query range) and the query
 * tiles that can see it. Produced by segpaged_mass_plan; the fields are private. 64 bytes. */
typedef struct {
  int32_t v[16];
} segpaged_mass_item;

/* Plans segpaged_token_mass (host only). Inputs as for segpaged_prefill_plan. Writes the items to
 * `items` (host, capacity entries; NULL to only count) and returns their number, or an error
 * (SEGPAGED_ERR_CAPACITY if capacity is too small). */
int64_t segpaged_mass_plan(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                           const segpaged_head_class* cls, const int32_t* page_table_offs,
                           segpaged_mass_item* items, int64_t capacity);

/* Device workspace segpaged_token_mass needs: a few partial sums per (KV head, query row) and a counter. */
size_t segpaged_mass_workspace_bytes(const segpaged_dims* dims, int32_t total_q);

/*
 * mass[r] for every query row r (dev, float32 [total_q]), as defined above. Recomputes the logits of
 * every (query tile, key tile) pair whose keys lie in the query range on the tensor cores and
 * normalises them with `lse`, the natural-log LSE [Hq, total_q] (dev, float32) that
 * segpaged_attn_prefill wrote for the same q, pools and scale. Same q, pools, page table and scale
 * as that prefill. items (dev) [num_items] from segpaged_mass_plan; workspace (dev, 256-byte
 * aligned) of segpaged_mass_workspace_bytes. frag_offs, frag_start, frag_cos_sin (dev, all NULL or
 * all set): the fragments of a prefill run with segpaged_attn_prefill_rope, whose keys are re-aligned
 * the same way here. The sum over KV heads is taken in a fixed order, so the result does not depend on
 * scheduling or on the physical page ids. Asynchronous on `stream`.
 */
int segpaged_token_mass(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool,
                        const int32_t* page_table, int64_t page_table_len, const segpaged_mass_item* items,
                        int64_t num_items, const float* lse, float softmax_scale, const int32_t* frag_offs,
                        const int32_t* frag_start, const float* frag_cos_sin, float* mass, void* workspace,
                        size_t workspace_bytes, int32_t* status, void* stream);

/*
 * Top-k tokens of each sequence by mass (all device memory): for sequence b, the k_b = min(max(
 * k_per_seq[b], 0), Lq_b) rows of [cu_seqlens_q[b], cu_seqlens_q[b+1]) with the largest mass; among
 * equal values the lower row wins. The chosen global row indices are written in ascending order to
 * selected[off_b .. off_b + k_b), off_b = sum of k_c over c < b (size `selected` for the sum of all
 * k_b). mass must be finite and >= 0 (as segpaged_token_mass writes it). One block per sequence.
 */
int segpaged_select_topk(int32_t num_seqs, const float* mass, const int32_t* cu_seqlens_q, const int32_t* k_per_seq,
                         int32_t* selected, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SEGPAGED_H */
