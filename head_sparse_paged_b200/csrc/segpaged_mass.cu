// segpaged_mass.cu -- host side of the token-mass and top-k selection calls (see include/segpaged.h):
// the mass plan, argument checks, tensor maps and launches. Allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/segpaged.h"
#include "host_common.h"
#include "mass_sm100.cuh"
#include "plan.h"
#include "topk_kernel.cuh"

using namespace segpaged;
using namespace segpaged::host;

static_assert(sizeof(segpaged_mass_item) == M_NFIELDS * sizeof(int32_t), "mass item layout");

namespace {
constexpr size_t kMassCounterBytes = 256;
}

extern "C" int64_t segpaged_mass_plan(const segpaged_dims* dims, const int32_t* ctx_len, const int32_t* q_len,
                                      const segpaged_head_class* cls, const int32_t* page_table_offs,
                                      segpaged_mass_item* items, int64_t capacity) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const int B = dims->num_seqs, H = dims->num_kv_heads, P = dims->page_size;
  if (B > 0 && (!ctx_len || !q_len || !cls || !page_table_offs)) return SEGPAGED_ERR_NULL;
  if (B > 0 && page_table_offs[0] != 0) return SEGPAGED_ERR_PAGES;
  const int G = dims->num_q_heads / H;
  const int npos = 128 / G;
  std::vector<segpaged_mass_item> out;
  int32_t qrow = 0;
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
      if (Lq == 0) continue;
      for (int32_t x = q0 / 128; x <= (L - 1) / 128; ++x) {
        // keys of the query range in this tile: [jmin, jmax]; the query positions that see any of them
        const int32_t jmin = std::max(q0, x * 128), jmax = std::min(L - 1, x * 128 + 127);
        int64_t last = L - 1;
        if (!c.is_global && jmin >= c.sink) last = std::min<int64_t>(L - 1, (int64_t)jmax + c.window - 1);
        const int32_t t_lo = (jmin - q0) / npos, t_hi = (int32_t)((last - q0) / npos);
        segpaged_mass_item it;
        std::memset(&it, 0, sizeof(it));
        it.v[M_SEQ] = b;
        it.v[M_KVH] = k;
        it.v[M_TILE] = x;
        it.v[M_TOFF] = page_table_offs[bk];
        it.v[M_NSINK] = sp.n_sink;
        it.v[M_W0] = sp.w0;
        it.v[M_GLOBAL] = c.is_global ? 1 : 0;
        it.v[M_SINK] = c.is_global ? 0 : c.sink;
        it.v[M_WIN] = c.is_global ? 0 : c.window;
        it.v[M_Q0] = q0;
        it.v[M_L] = L;
        it.v[M_QROW0] = qrow;
        it.v[M_T0] = t_lo;
        it.v[M_NT] = t_hi - t_lo + 1;
        it.v[M_TOTAL] = sp.total;
        it.v[M_LQ] = Lq;
        out.push_back(it);
      }
    }
    qrow += Lq;
  }
  // Longest first, so the persistent grid finishes together.
  std::stable_sort(out.begin(), out.end(), [](const segpaged_mass_item& a, const segpaged_mass_item& b) {
    return a.v[M_NT] > b.v[M_NT];
  });
  const int64_t n = (int64_t)out.size();
  if (!items) return n;
  if (capacity < n) return SEGPAGED_ERR_CAPACITY;
  if (n) std::memcpy(items, out.data(), sizeof(segpaged_mass_item) * (size_t)n);
  return n;
}

extern "C" size_t segpaged_mass_workspace_bytes(const segpaged_dims* dims, int32_t total_q) {
  if (!dims || dims->num_kv_heads < 1 || total_q < 0) return kMassCounterBytes;
  return kMassCounterBytes +
         ((kMassWarpgroups * (size_t)dims->num_kv_heads * (size_t)total_q * sizeof(float) + 255) & ~(size_t)255);
}

namespace {
template <int D, int P>
int launch_mass(const CUtensorMap& tq, const CUtensorMap& tk, const MassParams& p, int grid, cudaStream_t st) {
  using C = MassCfg<D, P>;
  static std::atomic<bool> configured[kMaxDevices];   // per device; a race only repeats the call
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SEGPAGED_ERR_CUDA;
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(segpaged_mass_kernel<D, P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return SEGPAGED_ERR_CUDA;
    configured[dev].store(true, std::memory_order_release);
  }
  segpaged_mass_kernel<D, P><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, p);
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}
}  // namespace

extern "C" int segpaged_token_mass(const segpaged_dims* dims, const void* q, int32_t total_q, const void* k_pool,
                                   const int32_t* page_table, int64_t page_table_len, const segpaged_mass_item* items,
                                   int64_t num_items, const float* lse, float softmax_scale,
                                   const int32_t* frag_offs, const int32_t* frag_start, const float* frag_cos_sin,
                                   float* mass, void* workspace, size_t workspace_bytes, int32_t* status,
                                   void* stream) {
  int rc = check_dims(dims);
  if ((frag_offs || frag_start || frag_cos_sin) && !(frag_offs && frag_start && frag_cos_sin)) return SEGPAGED_ERR_NULL;
  if (frag_cos_sin && !aligned16(frag_cos_sin)) return SEGPAGED_ERR_ALIGN;
  if (rc) return rc;
  if (num_items < 0 || num_items > INT32_MAX || total_q < 0 || page_table_len < 0) return SEGPAGED_ERR_DIMS;
  if (total_q == 0) return SEGPAGED_OK;
  if (!mass || !workspace) return SEGPAGED_ERR_NULL;
  if (workspace_bytes < segpaged_mass_workspace_bytes(dims, total_q)) return SEGPAGED_ERR_CAPACITY;
  if (!aligned16(workspace) || !aligned16(mass)) return SEGPAGED_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part = reinterpret_cast<float*>(ws + kMassCounterBytes);
  const int D = dims->head_dim, P = dims->page_size, Hq = dims->num_q_heads;
  const int G = Hq / dims->num_kv_heads;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEGPAGED_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return SEGPAGED_ERR_CUDA;
  if (num_items > 0) {
    if (!q || !k_pool || !page_table || !items || !lse) return SEGPAGED_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(items)) return SEGPAGED_ERR_ALIGN;
    if (dims->num_pages < 1) return SEGPAGED_ERR_DIMS;
    CUtensorMap tq, tk;
    if (!encode_3d(&tq, q, D, Hq, (uint64_t)total_q, 64, G, 128 / G) ||
        !encode_3d(&tk, k_pool, D, P, (uint64_t)dims->num_pages, 64, P, 1))
      return SEGPAGED_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), st) != cudaSuccess) return SEGPAGED_ERR_CUDA;
    MassParams p;
    p.page_table = page_table;
    p.page_table_len = page_table_len;
    p.items = reinterpret_cast<const int32_t*>(items);
    p.num_items = (int32_t)num_items;
    p.counter = reinterpret_cast<int32_t*>(ws);
    p.status = status;
    p.lse = lse;
    p.part = part;
    p.total_q = total_q;
    p.num_q_heads = Hq;
    p.num_kv_heads = dims->num_kv_heads;
    p.num_pages = dims->num_pages;
    p.log2_group = log2_int(G);
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.frags = RopeFragments{frag_offs, frag_start, frag_cos_sin};
    const int grid = (int)std::min<int64_t>(num_items, sms);
    rc = SEGPAGED_ERR_DIMS;
#define SEGPAGED_LAUNCH(DD, PP) \
  if (D == DD && P == PP) rc = launch_mass<DD, PP>(tq, tk, p, grid, st);
    SEGPAGED_LAUNCH(128, 16)
    SEGPAGED_LAUNCH(128, 32)
    SEGPAGED_LAUNCH(128, 64)
    SEGPAGED_LAUNCH(128, 128)
    SEGPAGED_LAUNCH(64, 16)
    SEGPAGED_LAUNCH(64, 32)
    SEGPAGED_LAUNCH(64, 64)
    SEGPAGED_LAUNCH(64, 128)
#undef SEGPAGED_LAUNCH
    if (rc != SEGPAGED_OK) return rc;
  } else {
    // no items: every partial is zero
    if (cudaMemsetAsync(part, 0, kMassWarpgroups * (size_t)dims->num_kv_heads * total_q * sizeof(float), st) !=
        cudaSuccess)
      return SEGPAGED_ERR_CUDA;
  }
  const int blocks = (int)std::min<int64_t>((total_q + 255) / 256, (int64_t)sms * 8);
  mass_reduce_kernel<<<blocks, 256, 0, st>>>(part, mass, total_q, kMassWarpgroups * dims->num_kv_heads);
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}

extern "C" int segpaged_select_topk(int32_t num_seqs, const float* mass, const int32_t* cu_seqlens_q,
                                    const int32_t* k_per_seq, int32_t* selected, void* stream) {
  if (num_seqs < 0) return SEGPAGED_ERR_DIMS;
  if (num_seqs == 0) return SEGPAGED_OK;
  if (!mass || !cu_seqlens_q || !k_per_seq || !selected) return SEGPAGED_ERR_NULL;
  topk_select_kernel<<<num_seqs, kTopkThreads, 0, static_cast<cudaStream_t>(stream)>>>(mass, cu_seqlens_q, k_per_seq,
                                                                                      selected);
  return cudaGetLastError() == cudaSuccess ? SEGPAGED_OK : SEGPAGED_ERR_CUDA;
}
