// plan.h -- the SegPaged storage rule and the prefill work-unit layout, shared by the host planner
// (segpaged_prefill_plan, segpaged_pages_bytes) and the device kernels.
//
// Storage rule. Logical page n of a (sequence, KV head) holds tokens [n*P, n*P + P). A global head
// keeps every page of its context; a local head keeps only the pages of its sink tokens and of its
// recent window (bjdmk.com.cn, 二 "三大核心机制" item 3: local heads physically store only sink and
// recent-window KV pages). The window pages are those any served query (positions L-Lq .. L-1) can
// see in its window, i.e. the pages holding a token >= max(L - Lq - W + 1, 0). When the sink pages
// and the window pages meet or overlap, every page is stored and the head's table is simply indexed
// by logical page.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define SP_HD __host__ __device__ __forceinline__
#else
#define SP_HD static inline
#endif

namespace segpaged {

SP_HD int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// How the page table of one (sequence, KV head) maps to logical pages: table index t < n_sink holds
// logical page t; table index t >= n_sink holds logical page w0 + (t - n_sink).
struct Split {
  int32_t n_sink;
  int32_t w0;
  int32_t total;  // stored pages = table length
};

SP_HD Split storage_split(int32_t L, int32_t Lq, int32_t is_global, int32_t sink, int32_t window, int32_t P) {
  Split s;
  const int32_t n_all = (int32_t)ceil_div(L, P);
  s.n_sink = n_all;
  s.w0 = n_all;
  s.total = n_all;
  if (is_global) return s;
  const int32_t ns = (int32_t)ceil_div(sink < L ? sink : L, P);
  int64_t lo = (int64_t)L - Lq - window + 1;
  if (lo < 0) lo = 0;
  const int32_t w0 = (int32_t)(lo / P);
  if (w0 <= ns) return s;  // sink and window pages meet: everything is stored
  s.n_sink = ns;
  s.w0 = w0;
  s.total = ns + (n_all - w0);
  return s;
}

// Work unit: one (sequence, KV head) and up to 2 x 128/G consecutive query positions, all G query heads
// of the group: two 128-row tensor-core tiles that share every K/V tile. Its keys are the pages at list
// positions [0, a_n + b_n): list position x < a_n is table index x (sink part), list position
// x >= a_n is table index b0 + (x - a_n) (window part). KV tiles are groups of 128/P consecutive
// list positions, n_kv = ceil((a_n + b_n) / (128/P)) of them. A record runs KV tiles [t0, t0 + n_tiles):
// all of them, or one chunk when a long unit is split across CTAs; a chunk writes a partial result
// (O / l in fp32 and its LSE) into partial slot `part`, and a combine record later merges the chunks of a
// unit in chunk order. With at most 128/G valid positions the second query tile has no rows (`half`).
enum UnitField {
  U_QROW = 0,     // row of the first position in Q / O (index into the packed query rows)
  U_POS0 = 1,     // absolute position of the first row
  U_NPOS = 2,     // valid positions in this unit (<= 2 x 128/G)
  U_KVH = 3,      // KV head
  U_TOFF = 4,     // offset of the head's page table
  U_NSINK = 5,    // Split::n_sink
  U_W0 = 6,       // Split::w0
  U_GLOBAL = 7,
  U_SINK = 8,
  U_WIN = 9,
  U_AN = 10,
  U_B0 = 11,
  U_BN = 12,
  U_NTILES = 13,  // KV tiles this record runs; < 0 marks the end of the schedule inside the kernel
  U_TOTAL = 14,   // Split::total (table length)
  U_SEQ = 15,
  U_T0 = 16,      // first KV tile of this record
  U_PART = 17,    // partial slot written by a chunk of a split unit, -1 when the record writes O directly
  U_HALF = 18,    // 1 when the second query tile has no valid rows
  U_NSPLIT = 19,  // chunks of the unit (combine records)
  // Fused append-and-attend (segpaged_attn_prefill_append). The list above then holds only the pages with
  // a key before the query range (split at q0), forming tiles [0, n_old_tiles); tiles from n_old_tiles on
  // cover the new pages new0 .. new0 + n_new - 1, whose rows are read from the dense new K/V instead of
  // the pool. Keys are valid in an old tile only below `split_q0` and in a new tile only from it.
  U_NOLDT = 20,   // tiles over the page list; the rest are new-page tiles (== U_NTILES without append)
  U_NEW0 = 21,    // first new logical page
  U_NNEW = 22,    // new pages (0 without append)
  U_SPLITQ = 23,  // q0 with append, INT32_MAX without (every listed key is valid)
  U_CUQ = 24,     // packed row of the sequence's first query (row of key position q0 in the new K/V)
  U_NFIELDS = 32
};
// A combine record reuses U_QROW, U_NPOS, U_KVH, U_SEQ, U_HALF; U_PART is its first partial slot and
// U_NSPLIT the number of consecutive slots to merge.

}  // namespace segpaged
