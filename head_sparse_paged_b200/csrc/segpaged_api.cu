// segpaged_api.cu -- host side of the SegPagedAttention C ABI (see include/segpaged.h).
//
// Argument validation, the storage accounting (segpaged_pages_bytes), the RoPE table, the work
// planner (segpaged_prefill_plan, the SELECTVISIBLESTATE step), TMA tensor-map encoding and the
// kernel launches. The library allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <vector>

#include "../../include/segpaged.h"
#include "build_kernel.cuh"
#include "host_common.h"
#include "combine_kernel.cuh"
#include "plan.h"
#include "prefill_sm100.cuh"

using namespace segpaged;
using namespace segpaged::host;

extern "C" {

const char* segpaged_error_string(int code) {
  switch (code) {
    case SEGPAGED_OK: return "ok";
    case SEGPAGED_ERR_NULL: return "a required pointer is NULL";
    case SEGPAGED_ERR_DIMS: return "unsupported or inconsistent dims";
    case SEGPAGED_ERR_CLASS: return "head class out of range (sink < 0 or window < 1 for a local head)";
    case SEGPAGED_ERR_SEQ: return "bad sequence lengths (negative, or Lq > L)";
    case SEGPAGED_ERR_PAGES: return "page-table offsets disagree with the storage rule";
    case SEGPAGED_ERR_CAPACITY: return "output array too small";
    case SEGPAGED_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case SEGPAGED_ERR_ALIGN: return "a base pointer is not 16-byte aligned";
    case SEGPAGED_ERR_UNSUPPORTED: return "the plan splits units; this entry point needs a plan made with split_ctas = 0";
    default: return "unknown error";
  }
}

int64_t segpaged_pages_bytes(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                             const segpaged_head_class* cls, int64_t* dense_bytes, int32_t* pages_per_head) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->num_seqs > 0 && (!ctx_len || !q_len || !cls)) return SEGPAGED_ERR_NULL;
  const int B = dims->num_seqs, H = dims->num_kv_heads, P = dims->page_size;
  int64_t stored = 0, dense = 0;
  for (int b = 0; b < B; ++b) {
    if (ctx_len[b] < 0 || q_len[b] < 0 || q_len[b] > ctx_len[b]) return SEGPAGED_ERR_SEQ;
    for (int k = 0; k < H; ++k) {
      const segpaged_head_class& c = cls[b * H + k];
      if ((rc = check_class(c))) return rc;
      const Split s = storage_split(ctx_len[b], q_len[b], c.is_global, c.sink, c.window, P);
      stored += s.total;
      dense += ceil_div(ctx_len[b], P);
      if (pages_per_head) pages_per_head[b * H + k] = s.total;
    }
  }
  const int64_t unit = (int64_t)P * dims->head_dim * 2 /*K and V*/ * 2 /*bf16*/;
  if (dense_bytes) *dense_bytes = dense * unit;
  return stored * unit;
}

int segpaged_rope_cos_sin(double theta, const int32_t* deltas, int32_t num_seqs, int32_t head_dim, float* out) {
  if (num_seqs < 0 || head_dim < 2 || (head_dim & 1) || !(theta > 0.0)) return SEGPAGED_ERR_DIMS;
  if (num_seqs > 0 && (!deltas || !out)) return SEGPAGED_ERR_NULL;
  const int half = head_dim / 2;
  for (int b = 0; b < num_seqs; ++b)
    for (int d = 0; d < half; ++d) {
      const double inv_freq = std::pow(theta, -2.0 * d / head_dim);
      const double ang = (double)deltas[b] * inv_freq;
      out[((int64_t)b * half + d) * 2 + 0] = (float)std::cos(ang);
      out[((int64_t)b * half + d) * 2 + 1] = (float)std::sin(ang);
    }
  return SEGPAGED_OK;
}

int segpaged_build(const segpaged_dims* dims, const void* k_dense, const void* v_dense, const int32_t* cu_seqlens_k,
                   const int32_t* q_len, const segpaged_head_class* cls, const int32_t* page_table,
                   const int32_t* page_table_offs, const float* rope_cos_sin, void* k_pool, void* v_pool,
                   int32_t* status, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->num_seqs == 0) return SEGPAGED_OK;
  if (!k_dense || !v_dense || !cu_seqlens_k || !q_len || !cls || !page_table || !page_table_offs || !k_pool || !v_pool)
    return SEGPAGED_ERR_NULL;
  if (!aligned16(k_dense) || !aligned16(v_dense) || !aligned16(k_pool) || !aligned16(v_pool) ||
      (rope_cos_sin && !aligned16(rope_cos_sin)))
    return SEGPAGED_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  BuildParams p;
  p.k_dense = static_cast<const __nv_bfloat16*>(k_dense);
  p.v_dense = static_cast<const __nv_bfloat16*>(v_dense);
  p.cu_k = cu_seqlens_k;
  p.q_len = q_len;
  p.cls = reinterpret_cast<const int32_t*>(cls);
  p.table = page_table;
  p.offs = page_table_offs;
  p.cos_sin = rope_cos_sin;
  p.k_pool = static_cast<__nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(v_pool);
  p.status = status;
  p.B = dims->num_seqs;
  p.Hkv = dims->num_kv_heads;
  p.P = dims->page_size;
  p.num_pages = dims->num_pages;
  const int grid = std::max(1, device_sm_count(dev)) * 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dims->head_dim == 128) {
    if (rope_cos_sin) build_scatter_kernel<128, true><<<grid, 256, 0, st>>>(p);
    else build_scatter_kernel<128, false><<<grid, 256, 0, st>>>(p);
  } else {
    if (rope_cos_sin) build_scatter_kernel<64, true><<<grid, 256, 0, st>>>(p);
    else build_scatter_kernel<64, false><<<grid, 256, 0, st>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}

}  // extern "C"

namespace {
// Planner of segpaged_prefill_plan (append = false) and segpaged_prefill_plan_append (append = true).
int64_t plan_units(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                   const segpaged_head_class* cls, const int32_t* page_table_offs, int32_t split_ctas,
                   segpaged_unit* units, int64_t capacity, segpaged_plan_info* info, bool append) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int B = dims->num_seqs, H = dims->num_kv_heads, P = dims->page_size;
  if (B > 0 && (!ctx_len || !q_len || !cls || !page_table_offs)) return SEGPAGED_ERR_NULL;
  const int G = dims->num_q_heads / H;
  const int npos_tile = 128 / G;
  const int npos = 2 * npos_tile;   // a unit is two 128-row query tiles sharing their K/V tiles
  const int ppt = 128 / P;
  std::vector<segpaged_unit> out;
  int32_t qrow = 0;
  if (page_table_offs && page_table_offs[0] != 0) return SEGPAGED_ERR_PAGES;
  for (int b = 0; b < B; ++b) {
    const int32_t L = ctx_len[b], Lq = q_len[b];
    if (L < 0 || Lq < 0 || Lq > L) return SEGPAGED_ERR_SEQ;
    const int32_t q0 = L - Lq;
    for (int k = 0; k < H; ++k) {
      const int bk = b * H + k;
      const segpaged_head_class& c = cls[bk];
      if ((rc = check_class(c))) return rc;
      const Split sp = storage_split(L, Lq, c.is_global, c.sink, c.window, P);
      if (page_table_offs[bk + 1] - page_table_offs[bk] != sp.total) return SEGPAGED_ERR_PAGES;
      const bool merged = sp.n_sink == sp.total;
      for (int32_t t0 = 0; t0 < Lq; t0 += npos) {
        const int32_t r0 = q0 + t0, nv = std::min(npos, Lq - t0), r1 = r0 + nv - 1;
        int32_t a_n = 0, b0 = 0, b_n = 0, b_lp = 0;   // b_lp: logical page of the window part's first entry
        if (c.is_global) {
          b_n = r1 / P + 1;
        } else {
          a_n = (int32_t)ceil_div(std::min<int64_t>(c.sink, (int64_t)r1 + 1), P);
          const int32_t wlo = std::max<int64_t>((int64_t)r0 - c.window + 1, 0);
          const int32_t lp_lo = wlo / P, lp_hi = r1 / P;
          if (merged) {
            if (lp_lo <= a_n) {  // sink and window ranges meet: one range from page 0
              a_n = 0;
              b0 = 0;
              b_n = lp_hi + 1;
            } else {
              b0 = lp_lo;
              b_n = lp_hi - lp_lo + 1;
              b_lp = lp_lo;
            }
          } else {
            b0 = sp.n_sink + (lp_lo - sp.w0);
            b_n = lp_hi - lp_lo + 1;
            b_lp = lp_lo;
          }
        }
        // Append: keys before q0 come from the pool (the list truncated to pages holding such a key), keys
        // from q0 on from the new K/V, as tiles of consecutive logical pages new0 .. new0 + n_new - 1.
        int32_t new0 = 0, n_new = 0;
        if (append) {
          const int32_t qpages = (int32_t)ceil_div(q0, P);
          a_n = std::min(a_n, qpages);
          b_n = std::max(0, std::min(b_n, qpages - b_lp));
          const int32_t lo_new = (c.is_global || c.sink > q0) ? q0 : std::max(q0, r0 - c.window + 1);
          if (lo_new <= r1) {
            new0 = lo_new / P;
            n_new = r1 / P - new0 + 1;
          }
        }
        const int32_t n_old_tiles = (int32_t)ceil_div(a_n + b_n, ppt);
        segpaged_unit u;
        std::memset(&u, 0, sizeof(u));
        u.v[U_QROW] = qrow + t0;
        u.v[U_POS0] = r0;
        u.v[U_NPOS] = nv;
        u.v[U_KVH] = k;
        u.v[U_TOFF] = page_table_offs[bk];
        u.v[U_NSINK] = sp.n_sink;
        u.v[U_W0] = sp.w0;
        u.v[U_GLOBAL] = c.is_global ? 1 : 0;
        u.v[U_SINK] = c.is_global ? 0 : c.sink;
        u.v[U_WIN] = c.is_global ? 0 : c.window;
        u.v[U_AN] = a_n;
        u.v[U_B0] = b0;
        u.v[U_BN] = b_n;
        u.v[U_NTILES] = n_old_tiles + (int32_t)ceil_div(n_new, ppt);
        u.v[U_TOTAL] = sp.total;
        u.v[U_SEQ] = b;
        u.v[U_T0] = 0;
        u.v[U_PART] = -1;
        u.v[U_HALF] = nv <= npos_tile ? 1 : 0;
        u.v[U_NSPLIT] = 0;
        u.v[U_NOLDT] = n_old_tiles;
        u.v[U_NEW0] = new0;
        u.v[U_NNEW] = n_new;
        u.v[U_SPLITQ] = append ? q0 : INT32_MAX;
        u.v[U_CUQ] = qrow;
        out.push_back(u);
      }
    }
    qrow += Lq;
  }
  // Tensor work of a record: KV tiles x query tiles it runs.
  auto cost = [](const segpaged_unit& u) { return (int64_t)u.v[U_NTILES] * (u.v[U_HALF] ? 1 : 2); };
  // Split long units across CTAs when one unit alone would exceed a CTA's fair share of the work (short
  // query ranges, decode-like tiles). A unit longer than a target T is cut into near-equal chunks of at
  // least 4 KV tiles (at most 256 chunks); each chunk writes a partial result that the combine launch merges.
  // T is chosen by a cost model of the whole call, fitted to launches measured on this B200 (one cost unit, a KV
  // tile of one query tile, is about 1 us of the launch): the longest-first schedule of the records over the
  // CTAs with a fixed cost per record (claim, query load, pipeline ramp), plus the partial rows the chunks write
  // and the combine merges, plus the combine launch itself. Candidates run from one to four waves of equal
  // pieces up to no split at all, so short units are left whole when splitting them costs more than it saves.
  std::vector<segpaged_unit> groups;
  int32_t slots = 0;
  if (split_ctas > 0 && !out.empty()) {
    int64_t total = 0, longest = 0;
    for (const auto& u : out) {
      total += cost(u);
      longest = std::max(longest, cost(u));
    }
    if (longest * split_ctas > total) {
      auto chunk_of = [](const segpaged_unit& u, int64_t target) {
        const int32_t weight = u.v[U_HALF] ? 1 : 2;
        int32_t chunk = (int32_t)std::max<int64_t>(4, std::min<int64_t>(INT32_MAX, ceil_div(target, weight)));
        return std::max<int32_t>(chunk, (int32_t)ceil_div(u.v[U_NTILES], kCombineMaxSplit));
      };
      constexpr double kRecordCost = 6.0;      // per record, in cost units
      constexpr double kPartialRowCost = 3e-4; // per partial row (written by a chunk, read by the combine)
      constexpr double kCombineCost = 4.0;     // the combine launch, when anything is split
      auto model = [&](int64_t target) {
        std::vector<int64_t> items;
        int64_t rows = 0;
        for (const auto& u : out) {
          const int32_t n = u.v[U_NTILES], chunk = chunk_of(u, target), weight = u.v[U_HALF] ? 1 : 2;
          if (n <= chunk) {
            items.push_back(cost(u));
            continue;
          }
          const int32_t k = (int32_t)ceil_div(n, chunk);
          for (int32_t c = 0; c < k; ++c) items.push_back((int64_t)(n / k + (c < n % k ? 1 : 0)) * weight);
          rows += (int64_t)k * u.v[U_NPOS] * G;
        }
        std::sort(items.begin(), items.end(), std::greater<int64_t>());
        std::priority_queue<double, std::vector<double>, std::greater<double>> load;
        for (int32_t c = 0; c < split_ctas; ++c) load.push(0.0);
        double span = 0.0;
        for (int64_t it : items) {
          const double x = load.top() + (double)it + kRecordCost;
          load.pop();
          load.push(x);
          span = std::max(span, x);
        }
        return span + (rows > 0 ? kCombineCost + kPartialRowCost * (double)rows : 0.0);
      };
      std::vector<int64_t> targets;
      for (int waves = 4; waves >= 1; --waves) targets.push_back(ceil_div(total, (int64_t)waves * split_ctas));
      for (int64_t t = targets.back(); t < longest;) {
        t = std::max<int64_t>(t + 1, t * 5 / 4);
        targets.push_back(std::min(t, longest));    // the last candidate splits nothing
      }
      int64_t best_target = longest;
      double best_time = model(longest);
      for (int64_t t : targets) {   // ties keep the coarser split (less partial traffic): candidates ascend
        const double x = model(t);
        if (x < best_time - 1e-9 || (x <= best_time + 1e-9 && t > best_target)) {
          best_time = x;
          best_target = t;
        }
      }
      std::vector<segpaged_unit> work;
      for (const auto& u : out) {
        const int32_t n = u.v[U_NTILES];
        const int32_t chunk = chunk_of(u, best_target);
        if (n <= chunk) {
          work.push_back(u);
          continue;
        }
        const int32_t k = (int32_t)ceil_div(n, chunk);
        segpaged_unit g = u;
        g.v[U_PART] = slots;
        g.v[U_NSPLIT] = k;
        g.v[U_NTILES] = 0;
        groups.push_back(g);
        int32_t t0 = 0;
        for (int32_t c = 0; c < k; ++c) {
          const int32_t len = n / k + (c < n % k ? 1 : 0);
          segpaged_unit w = u;
          w.v[U_T0] = t0;
          w.v[U_NTILES] = len;
          w.v[U_PART] = slots++;
          work.push_back(w);
          t0 += len;
        }
      }
      out.swap(work);
    }
  }
  // Longest first, so the persistent grid finishes together -- but by cost bucket (16 levels relative to
  // the longest record), keeping the plan order (sequence, KV head, query tile, chunk) inside a bucket.
  // CTAs that start together then mostly work on the same head and sweep its pages in step, so a page is
  // fetched from HBM once and served from L2 to the other CTAs, instead of every CTA streaming another head.
  int64_t max_cost = 1;
  for (const auto& u : out) max_cost = std::max(max_cost, cost(u));
  auto bucket = [&](const segpaged_unit& u) { return (cost(u) * 16 + max_cost / 2) / max_cost; };
  std::stable_sort(out.begin(), out.end(),
                   [&](const segpaged_unit& a, const segpaged_unit& b) { return bucket(a) > bucket(b); });
  if (info) {
    info->total_q = qrow;
    info->page_table_len = B > 0 ? page_table_offs[B * H] : 0;
    info->num_q_heads = dims->num_q_heads;
    info->num_kv_heads = H;
    info->head_dim = dims->head_dim;
    info->page_size = P;
    info->num_units = (int64_t)out.size();
    info->num_groups = (int64_t)groups.size();
    info->num_partials = slots;
    info->num_half_units = 0;
    for (const auto& u : out) info->num_half_units += u.v[U_HALF] ? 1 : 0;
    info->combine_row_blocks = 0;
    for (const auto& g : groups)
      info->combine_row_blocks =
          std::max(info->combine_row_blocks, combine_blocks_of(g.v[U_NPOS], g.v[U_NSPLIT], G));
  }
  out.insert(out.end(), groups.begin(), groups.end());
  const int64_t n = (int64_t)out.size();
  if (!units) return n;
  if (capacity < n) return SEGPAGED_ERR_CAPACITY;
  if (n) std::memcpy(units, out.data(), sizeof(segpaged_unit) * (size_t)n);
  return n;
}
}  // namespace

extern "C" {

int segpaged_rope_realign(const segpaged_dims* dims, const int32_t* cu_seqlens_k, const int32_t* q_len,
                          const segpaged_head_class* cls, const int32_t* page_table, const int32_t* page_table_offs,
                          const int32_t* frag_offs, const int32_t* frag_start, const float* frag_cos_sin,
                          const void* k_pool, void* k_pool_out, int32_t* status, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->num_seqs == 0) return SEGPAGED_OK;
  if (!cu_seqlens_k || !q_len || !cls || !page_table || !page_table_offs || !frag_offs || !frag_start ||
      !frag_cos_sin || !k_pool || !k_pool_out)
    return SEGPAGED_ERR_NULL;
  if (k_pool == k_pool_out) return SEGPAGED_ERR_DIMS;
  if (!aligned16(k_pool) || !aligned16(k_pool_out) || !aligned16(frag_cos_sin)) return SEGPAGED_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  RealignParams p;
  p.k_in = static_cast<const __nv_bfloat16*>(k_pool);
  p.k_out = static_cast<__nv_bfloat16*>(k_pool_out);
  p.cu_k = cu_seqlens_k;
  p.q_len = q_len;
  p.cls = reinterpret_cast<const int32_t*>(cls);
  p.table = page_table;
  p.offs = page_table_offs;
  p.frags = RopeFragments{frag_offs, frag_start, frag_cos_sin};
  p.status = status;
  p.B = dims->num_seqs;
  p.Hkv = dims->num_kv_heads;
  p.P = dims->page_size;
  p.num_pages = dims->num_pages;
  const int grid = std::max(1, device_sm_count(dev)) * 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dims->head_dim == 128) rope_realign_kernel<128><<<grid, 256, 0, st>>>(p);
  else rope_realign_kernel<64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}

int64_t segpaged_prefill_plan(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                              const segpaged_head_class* cls, const int32_t* page_table_offs, int32_t split_ctas,
                              segpaged_unit* units, int64_t capacity, segpaged_plan_info* info) {
  return plan_units(dims, ctx_len, q_len, cls, page_table_offs, split_ctas, units, capacity, info, false);
}

int64_t segpaged_prefill_plan_append(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                                     const segpaged_head_class* cls, const int32_t* page_table_offs,
                                     int32_t split_ctas, segpaged_unit* units, int64_t capacity,
                                     segpaged_plan_info* info) {
  return plan_units(dims, ctx_len, q_len, cls, page_table_offs, split_ctas, units, capacity, info, true);
}

namespace {
constexpr size_t kCounterBytes = 256;
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t partial_o_bytes(int64_t slots, int D) { return align256((size_t)slots * 256 * D * sizeof(float)); }
}  // namespace

size_t segpaged_prefill_workspace_bytes(const segpaged_dims* dims, const segpaged_plan_info* info) {
  if (!dims || !info || info->num_partials < 0) return kCounterBytes;
  return kCounterBytes + partial_o_bytes(info->num_partials, dims->head_dim) +
         align256((size_t)info->num_partials * 256 * sizeof(float));
}

}  // extern "C"

namespace {

template <int D, int P, int MODE, int HALF>
int launch_prefill_v(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkn,
                     const CUtensorMap& tvn, const PrefillParams& p, int grid, cudaStream_t st) {
  using C = PrefillCfg<D, P, MODE == kModeRope>;
  static std::atomic<bool> configured[kMaxDevices];   // per device; a race only repeats the call
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SEGPAGED_ERR_CUDA;
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(segpaged_prefill_kernel<D, P, MODE, HALF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return SEGPAGED_ERR_CUDA;
    configured[dev].store(true, std::memory_order_release);
  }
  segpaged_prefill_kernel<D, P, MODE, HALF><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, tkn, tvn, p);
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}

// The shared-half variant when the plan has half units (rows in one query tile only); for the plain kernel
// with half units only, the variant that turns the unused second query buffer into one more K/V slot.
template <int D, int P, int MODE>
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkn,
                   const CUtensorMap& tvn, const PrefillParams& p, int grid, cudaStream_t st, int half) {
  if constexpr (MODE == kModePlain) {
    if (half == 2) return launch_prefill_v<D, P, MODE, 2>(tq, tk, tv, tkn, tvn, p, grid, st);
  }
  return half ? launch_prefill_v<D, P, MODE, 1>(tq, tk, tv, tkn, tvn, p, grid, st)
              : launch_prefill_v<D, P, MODE, 0>(tq, tk, tv, tkn, tvn, p, grid, st);
}

}  // namespace

template <int D>
int launch_combine(const CombineParams& c, cudaStream_t st) {
  if (c.num_groups <= 0) return SEGPAGED_OK;
  // records x row blocks of 32 rows (as many as the widest record needs) x 8 column ranges (used by records
  // of more than 16 chunks), in stream order after the prefill. (As a programmatic dependent launch, with its
  // blocks resident before the prefill's last CTAs finish and a grid-dependency wait in the kernel, every
  // split workload measured 1-4 % slower.)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<int64_t>(c.num_groups, 65535), (unsigned)c.row_blocks, 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  if (cudaLaunchKernelEx(&cfg, segpaged_combine_kernel<D>, c) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}

namespace {
int attn_prefill(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool, const void* v_pool,
                 const int32_t* page_table, int64_t page_table_len, const segpaged_unit* plan,
                 const segpaged_plan_info* info, float softmax_scale, const RopeFragments* frags, const void* k_new,
                 const void* v_new, void* o, float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                 void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!info) return SEGPAGED_ERR_NULL;
  const int64_t num_units = info->num_units;
  if (num_units < 0 || info->num_groups < 0 || info->num_partials < 0 || total_q < 0 || page_table_len < 0 ||
      num_units > INT32_MAX || info->num_groups > INT32_MAX)
    return SEGPAGED_ERR_DIMS;
  if (num_units == 0) return SEGPAGED_OK;
  if (!q || !k_pool || !v_pool || !page_table || !plan || !o || !lse || !workspace) return SEGPAGED_ERR_NULL;
  // the plan must have been made for this call's shape: its records address rows, heads and table entries
  if (info->total_q != total_q || info->num_q_heads != dims->num_q_heads || info->num_kv_heads != dims->num_kv_heads ||
      info->head_dim != dims->head_dim || info->page_size != dims->page_size || page_table_len < info->page_table_len ||
      info->num_half_units < 0 || info->num_half_units > num_units || (info->num_groups > 0) != (info->num_partials > 0))
    return SEGPAGED_ERR_DIMS;
  if (workspace_bytes < segpaged_prefill_workspace_bytes(dims, info)) return SEGPAGED_ERR_CAPACITY;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o) || !aligned16(plan) ||
      !aligned16(workspace))
    return SEGPAGED_ERR_ALIGN;
  if (total_q < 1 || dims->num_pages < 1) return SEGPAGED_ERR_DIMS;
  const int D = dims->head_dim, P = dims->page_size, Hq = dims->num_q_heads;
  const int G = Hq / dims->num_kv_heads;
  const bool append = k_new != nullptr;
  if (append && (!aligned16(k_new) || !aligned16(v_new))) return SEGPAGED_ERR_ALIGN;
  CUtensorMap tq, tk, tv, tkn, tvn;
  if (!encode_3d(&tq, q, D, Hq, (uint64_t)total_q, 64, G, 128 / G) ||
      !encode_3d(&tk, k_pool, D, P, (uint64_t)dims->num_pages, 64, P, 1) ||
      !encode_3d(&tv, v_pool, D, P, (uint64_t)dims->num_pages, 64, P, 1))
    return SEGPAGED_ERR_CUDA;
  // new K/V [total_q, Hkv, D]: P-row boxes of one KV head, the same shared-memory layout as a pool page
  if (append) {
    if (!encode_3d(&tkn, k_new, D, dims->num_kv_heads, (uint64_t)total_q, 64, 1, P) ||
        !encode_3d(&tvn, v_new, D, dims->num_kv_heads, (uint64_t)total_q, 64, 1, P))
      return SEGPAGED_ERR_CUDA;
  } else {
    tkn = tk;
    tvn = tv;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return SEGPAGED_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = (int)std::min<int64_t>(num_units, sms);
  // the work counter is read only when some CTA claims a second unit
  if (num_units > grid && cudaMemsetAsync(workspace, 0, sizeof(int32_t), st) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PrefillParams p;
  p.page_table = page_table;
  p.page_table_len = page_table_len;
  p.units = reinterpret_cast<const int32_t*>(plan);
  p.num_units = (int32_t)num_units;
  p.counter = reinterpret_cast<int32_t*>(ws);
  p.status = status;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.part_o = reinterpret_cast<float*>(ws + kCounterBytes);
  p.part_lse = reinterpret_cast<float*>(ws + kCounterBytes + partial_o_bytes(info->num_partials, D));
  p.total_q = total_q;
  p.num_q_heads = Hq;
  p.num_partials = (int32_t)std::min<int64_t>(info->num_partials, INT32_MAX);
  p.num_seqs = dims->num_seqs;
  p.num_pages = dims->num_pages;
  p.log2_group = log2_int(G);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.frags = frags ? *frags : RopeFragments{nullptr, nullptr, nullptr};
  // 0: no half units; 1: some; 2: all of them
  const int half = info->num_half_units <= 0 ? 0 : (info->num_half_units >= num_units ? 2 : 1);
  p.append = append ? 1 : 0;
  p.num_kv_heads = dims->num_kv_heads;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_pool = static_cast<__nv_bfloat16*>(const_cast<void*>(k_pool));
  p.v_pool = static_cast<__nv_bfloat16*>(const_cast<void*>(v_pool));
  rc = SEGPAGED_ERR_DIMS;
#define SEGPAGED_LAUNCH(DD, PP)                                                   \
  if (D == DD && P == PP)                                                          \
    rc = frags    ? launch_prefill<DD, PP, kModeRope>(tq, tk, tv, tkn, tvn, p, grid, st, half)   \
         : append ? launch_prefill<DD, PP, kModeAppend>(tq, tk, tv, tkn, tvn, p, grid, st, half) \
                  : launch_prefill<DD, PP, kModePlain>(tq, tk, tv, tkn, tvn, p, grid, st, half);
  SEGPAGED_LAUNCH(128, 16)
  SEGPAGED_LAUNCH(128, 32)
  SEGPAGED_LAUNCH(128, 64)
  SEGPAGED_LAUNCH(128, 128)
  SEGPAGED_LAUNCH(64, 16)
  SEGPAGED_LAUNCH(64, 32)
  SEGPAGED_LAUNCH(64, 64)
  SEGPAGED_LAUNCH(64, 128)
#undef SEGPAGED_LAUNCH
  if (rc != SEGPAGED_OK || info->num_groups == 0) return rc;
  CombineParams c;
  c.records = reinterpret_cast<const int32_t*>(plan) + num_units * U_NFIELDS;
  c.num_groups = (int32_t)info->num_groups;
  c.part_o = p.part_o;
  c.part_lse = p.part_lse;
  c.o = p.o;
  c.lse = lse;
  c.total_q = total_q;
  c.num_q_heads = Hq;
  c.num_partials = p.num_partials;
  c.log2_group = p.log2_group;
  c.status = status;
  const int64_t rb = info->combine_row_blocks;
  c.row_blocks = (rb > 0 && rb < kCombineRows / kCombineBlockRows) ? (int32_t)rb : kCombineRows / kCombineBlockRows;
  return D == 128 ? launch_combine<128>(c, st) : launch_combine<64>(c, st);
}
}  // namespace

extern "C" int segpaged_attn_prefill(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool,
                                     const void* v_pool, const int32_t* page_table, int64_t page_table_len,
                                     const segpaged_unit* plan, const segpaged_plan_info* info, float softmax_scale,
                                     void* o, float* lse, void* workspace, size_t workspace_bytes, int32_t* status,
                                     void* stream) {
  return attn_prefill(dims, q, total_q, k_pool, v_pool, page_table, page_table_len, plan, info, softmax_scale, nullptr,
                      nullptr, nullptr, o, lse, workspace, workspace_bytes, status, stream);
}

extern "C" int segpaged_attn_prefill_append(const segpaged_dims* dims, const void* q, int32_t total_q,
                                            const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                            const int32_t* page_table, int64_t page_table_len,
                                            const segpaged_unit* plan, const segpaged_plan_info* info,
                                            float softmax_scale, void* o, float* lse, void* workspace,
                                            size_t workspace_bytes, int32_t* status, void* stream) {
  if (info && info->num_units > 0 && (!k_new || !v_new)) return SEGPAGED_ERR_NULL;
  return attn_prefill(dims, q, total_q, k_pool, v_pool, page_table, page_table_len, plan, info, softmax_scale, nullptr,
                      k_new, v_new, o, lse, workspace, workspace_bytes, status, stream);
}

extern "C" int segpaged_attn_prefill_rope(const segpaged_dims* dims, const void* q, int32_t total_q,
                                          const void* k_pool, const void* v_pool, const int32_t* page_table,
                                          int64_t page_table_len, const segpaged_unit* plan,
                                          const segpaged_plan_info* info, float softmax_scale,
                                          const int32_t* frag_offs, const int32_t* frag_start,
                                          const float* frag_cos_sin, void* o, float* lse, void* workspace,
                                          size_t workspace_bytes, int32_t* status, void* stream) {
  if (!frag_offs || !frag_start || !frag_cos_sin) return SEGPAGED_ERR_NULL;
  if (!aligned16(frag_cos_sin)) return SEGPAGED_ERR_ALIGN;
  const RopeFragments f{frag_offs, frag_start, frag_cos_sin};
  return attn_prefill(dims, q, total_q, k_pool, v_pool, page_table, page_table_len, plan, info, softmax_scale, &f,
                      nullptr, nullptr, o, lse, workspace, workspace_bytes, status, stream);
}

// ------------------------------------------------------------------------------------------------
// Allocation-free prefill entry point.
//
// Some callers cannot allocate device memory when they run prefill -- for example code running under
// a framework's own memory pool, or a runtime that forbids allocation on its request path -- so they
// cannot provide the work-unit list and the work-counter workspace that segpaged_attn_prefill needs.
// For them, both live in one file-scope device array below. Every GPU that loads this library holds
// it (2 MiB) until the process exits. All calls on a device share it and it keeps the last call's
// contents, so the counter is cleared by every call that reads it; calls whose work overlaps on the
// GPU race on it.
// ------------------------------------------------------------------------------------------------
namespace {
constexpr int64_t kNoAllocMaxUnits = 16384;   // the most work units one call accepts
constexpr int64_t kNoAllocUnitOffset = 64;    // int32 words before the unit list (counter in word 0)
}  // namespace

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocUnitOffset + kNoAllocMaxUnits * U_NFIELDS];

namespace {
std::mutex g_noalloc_mutex;
int32_t* g_noalloc_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device. In host code the array's name is only a
// host-side stand-in, so its address is looked up once per device, with that device current.
int noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SEGPAGED_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SEGPAGED_ERR_CUDA;
    g_noalloc_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_addr[dev];
  return SEGPAGED_OK;
}
}  // namespace

extern "C" int segpaged_attn_prefill_noalloc(const segpaged_dims* dims, const void* q, int32_t total_q,
                                             const void* k_pool, const void* v_pool, const int32_t* page_table,
                                             int64_t page_table_len, const segpaged_unit* units_host,
                                             int64_t num_units, float softmax_scale, void* o, float* lse,
                                             int32_t* status, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (num_units < 0) return SEGPAGED_ERR_DIMS;
  if (num_units > kNoAllocMaxUnits) return SEGPAGED_ERR_CAPACITY;
  if (num_units == 0) return SEGPAGED_OK;
  if (!units_host) return SEGPAGED_ERR_NULL;
  // The static array holds no partial results, so split plans (chunks or combine records) are refused.
  for (int64_t i = 0; i < num_units; ++i)
    if (units_host[i].v[U_PART] >= 0 || units_host[i].v[U_NSPLIT] > 0) return SEGPAGED_ERR_UNSUPPORTED;
  // Every unit must stay inside this call's arrays: its rows in [0, total_q), its KV head in [0, Hkv), its
  // page-table entries in [0, page_table_len), at most two query tiles of positions.
  const int32_t npos_tile = 128 / (dims->num_q_heads / dims->num_kv_heads);
  for (int64_t i = 0; i < num_units; ++i) {
    const int32_t* u = units_host[i].v;
    const int32_t cap = u[U_HALF] ? npos_tile : 2 * npos_tile;
    if (u[U_QROW] < 0 || u[U_NPOS] < 0 || u[U_NPOS] > cap || (int64_t)u[U_QROW] + u[U_NPOS] > total_q ||
        u[U_KVH] < 0 || u[U_KVH] >= dims->num_kv_heads || u[U_TOFF] < 0 || u[U_TOTAL] < 0 ||
        (int64_t)u[U_TOFF] + u[U_TOTAL] > page_table_len || u[U_NTILES] < 0 || u[U_T0] != 0 || u[U_NNEW] != 0)
      return SEGPAGED_ERR_DIMS;
  }
  int32_t* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  int32_t* units_dev = scratch + kNoAllocUnitOffset;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(units_dev, units_host, sizeof(segpaged_unit) * (size_t)num_units, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SEGPAGED_ERR_CUDA;
  // The work counter (word 0) is zeroed on the stream before a launch that claims units from it.
  segpaged_plan_info info;
  info.num_units = num_units;
  info.num_groups = 0;
  info.num_partials = 0;
  info.num_half_units = 0;
  for (int64_t i = 0; i < num_units; ++i) info.num_half_units += units_host[i].v[U_HALF] ? 1 : 0;
  info.combine_row_blocks = 0;
  info.total_q = total_q;
  info.page_table_len = page_table_len;
  info.num_q_heads = dims->num_q_heads;
  info.num_kv_heads = dims->num_kv_heads;
  info.head_dim = dims->head_dim;
  info.page_size = dims->page_size;
  return segpaged_attn_prefill(dims, q, total_q, k_pool, v_pool, page_table, page_table_len,
                               reinterpret_cast<const segpaged_unit*>(units_dev), &info, softmax_scale, o, lse,
                               scratch, kNoAllocUnitOffset * sizeof(int32_t), status, stream);
}
