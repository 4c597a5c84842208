// prefill_sm100.cuh -- EXECUTE: SegPagedAttention prefill on B200 (sm_100a).
//
// One persistent kernel runs every query head over exactly its own ragged, paged KV with no mask
// tensor (zhichai.net, 事件内容 item 3; bjdmk.com.cn, 二 item 3; aiboss88.com, 技術原則, item on paged
// storage removing the attn_mask penalty). Visibility: key j is visible to query position i iff
// j <= i and (global head, or j < S, or j > i - W).
//
// Work: units of (sequence, KV head, up to 128/G query positions x G query heads = 128 tile rows),
// planned on the host with their visible page ranges and sorted longest-first; CTAs (one per SM)
// claim them through a global atomic counter.
//
// Per CTA, 6 warps:
//   warp 0   producer: claims units, TMA-loads the Q tile (3-D map over [rows, Hq, D], box 64 x G x
//            128/G) and, for every 128-key tile, the K and V pages (3-D map over [pages, P, D],
//            coordinate = physical page id) into 128B-swizzled shared-memory slots.
//   warp 1   MMA issuer: S = Q K^T (tcgen05.mma, both operands from shared memory, f32 in TMEM,
//            double-buffered) and O += P V (P read from TMEM, V MN-major from shared memory).
//   warps 2-5 softmax: one tile row per thread. tcgen05.ld of the S row, per-row bounds only on
//            edge tiles, row max, lazy O rescale (only when the running max grows by more than
//            2^8), exp2, row sum, P written back to TMEM as bf16 over the S buffer, and the
//            epilogue (O / l -> bf16, LSE = ln 2 * (m + log2 l)).
// Every wait is bounded: on a timeout the CTA raises its abort flag, reports
// SEGPAGED_STATUS_TIMEOUT, drains the MMA pipe and frees its tensor memory before returning.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"
#include "sm100_ptx.cuh"

namespace segpaged {

constexpr int32_t kStatusPageId = 1;
constexpr int32_t kStatusTimeout = 4;
constexpr int32_t kStatusUnit = 8;

template <int D, int P>
struct PrefillCfg {
  static constexpr int BM = 128;                 // tile rows (positions x heads)
  static constexpr int BN = 128;                 // keys per KV tile
  static constexpr int NH = D / 64;              // 128-byte swizzle column blocks across D
  static constexpr int BLK = BN * 128;           // bytes of one 64-column block of a 128-row tile
  static constexpr int TILE_BYTES = BN * D * 2;  // one K or V tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int NSLOT = (D == 128) ? 5 : 10;
  static constexpr int PPT = BN / P;             // pages per KV tile
  static constexpr int SMEM_BYTES = 2 * Q_BYTES + NSLOT * TILE_BYTES + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;     // S0 [0,128) S1 [128,256) O [256, 256+D)
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t IDESC_O = ptx::idesc_bf16_f32(128, D, 0, 1);
};

struct PrefillParams {
  const int32_t* page_table;
  int64_t page_table_len;
  const int32_t* units;  // [num_units][U_NFIELDS]
  int32_t num_units;
  int32_t* counter;      // zeroed before the launch
  int32_t* status;       // nullable
  __nv_bfloat16* o;      // [total_q, Hq, D]
  float* lse;            // [Hq, total_q]
  int32_t total_q, num_q_heads, num_pages, log2_group;
  float scale_log2;      // softmax_scale * log2(e)
};

struct PrefillShared {
  uint64_t unit_full[2], unit_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_free, mma_drain;
  uint64_t kv_full[10], kv_empty[10];
  __align__(16) int32_t unit[2][U_NFIELDS];
  uint32_t tmem_base;
  int abort;
};

// List position x of a unit -> page-table index.
__device__ __forceinline__ int32_t unit_table_index(const int32_t* u, int32_t x) {
  return x < u[U_AN] ? x : u[U_B0] + (x - u[U_AN]);
}
// Page-table index -> logical page.
__device__ __forceinline__ int32_t unit_logical_page(const int32_t* u, int32_t idx) {
  return idx < u[U_NSINK] ? idx : u[U_W0] + (idx - u[U_NSINK]);
}

template <int D, int P>
__global__ void __launch_bounds__(192, 1)
    segpaged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PrefillCfg<D, P>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrefillShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                        // 2 x Q_BYTES
  uint8_t* sKV = smem + 2 * C::Q_BYTES;      // NSLOT x TILE_BYTES
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sh.abort;
  int32_t* status = p.status;

  // ---------------------------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.unit_full[i], 1);
      ptx::mbar_init(&sh.unit_empty[i], 5);   // MMA lane 0 + 4 softmax warps
      ptx::mbar_init(&sh.q_full[i], 1);
      ptx::mbar_init(&sh.q_empty[i], 1);
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.p_full[i], 4);
      ptx::mbar_init(&sh.pv_done[i], 1);
    }
    ptx::mbar_init(&sh.o_free, 4);
    ptx::mbar_init(&sh.mma_drain, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      ptx::mbar_init(&sh.kv_full[i], 1);
      ptx::mbar_init(&sh.kv_empty[i], 1);
    }
    sh.abort = 0;
    ptx::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // KV slots start zeroed: a partial tile leaves earlier (finite) data in the rows it does not
  // load, and those columns are masked, so their probability is exactly 0.
  for (int x = threadIdx.x; x < C::NSLOT * C::TILE_BYTES / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(sKV)[x] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t tS = tmem, tO = tmem + 256;
  const int G = 1 << p.log2_group;

  if (warp == 0) {
    // ------------------------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_item = 0, qcnt = 0;
      for (uint32_t ring = 0;; ++ring) {
        const int32_t u = atomicAdd(p.counter, 1);
        const int slot = ring & 1;
        if (!ptx::mbar_wait(&sh.unit_empty[slot], ((ring >> 1) & 1) ^ 1, abort, status, kStatusTimeout)) break;
        const bool done = u >= p.num_units;
        int32_t* U = sh.unit[slot];
        if (done) {
          U[U_NTILES] = -1;
        } else {
          const int4* src = reinterpret_cast<const int4*>(p.units + (int64_t)u * U_NFIELDS);
#pragma unroll
          for (int i = 0; i < U_NFIELDS / 4; ++i) reinterpret_cast<int4*>(U)[i] = src[i];
        }
        ptx::mbar_arrive(&sh.unit_full[slot]);
        if (done) break;
        const int qb = qcnt & 1;
        if (!ptx::mbar_wait(&sh.q_empty[qb], ((qcnt >> 1) & 1) ^ 1, abort, status, kStatusTimeout)) break;
        ptx::mbar_arrive_expect_tx(&sh.q_full[qb], C::Q_BYTES);
#pragma unroll
        for (int h = 0; h < C::NH; ++h)
          ptx::tma_load_3d(sQ + qb * C::Q_BYTES + h * C::BLK, &tm_q, h * 64, U[U_KVH] * G, U[U_QROW], &sh.q_full[qb]);
        ++qcnt;
        const int32_t npages = U[U_AN] + U[U_BN];
        const int32_t ntiles = U[U_NTILES];
        const int64_t toff = U[U_TOFF];
        bool ok = true;
        for (int32_t t = 0; t < ntiles && ok; ++t) {
          int32_t pages[C::PPT];
          int32_t n_ok = 0;
#pragma unroll
          for (int c = 0; c < C::PPT; ++c) {
            const int32_t x = t * C::PPT + c;
            pages[c] = -1;
            if (x < npages) {
              const int32_t idx = unit_table_index(U, x);
              int32_t pid = 0;
              if (idx < 0 || idx >= U[U_TOTAL] || toff + idx >= p.page_table_len) {
                if (status) atomicOr(status, kStatusUnit);
              } else {
                pid = p.page_table[toff + idx];
                if (pid < 0 || pid >= p.num_pages) {
                  if (status) atomicOr(status, kStatusPageId);
                  pid = 0;
                }
              }
              pages[c] = pid;
              ++n_ok;
            }
          }
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const int s = kv_item % C::NSLOT;
            if (!ptx::mbar_wait(&sh.kv_empty[s], ((kv_item / C::NSLOT) & 1) ^ 1, abort, status, kStatusTimeout)) {
              ok = false;
              break;
            }
            ptx::mbar_arrive_expect_tx(&sh.kv_full[s], (uint32_t)(n_ok * P * D * 2));
            uint8_t* dst = sKV + s * C::TILE_BYTES;
#pragma unroll
            for (int c = 0; c < C::PPT; ++c) {
              if (pages[c] < 0) continue;
#pragma unroll
              for (int h = 0; h < C::NH; ++h)
                ptx::tma_load_3d(dst + h * C::BLK + c * P * 128, which ? &tm_v : &tm_k, h * 64, 0, pages[c],
                                 &sh.kv_full[s]);
            }
            ++kv_item;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t q_base = ptx::smem_addr(sQ), kv_base = ptx::smem_addr(sKV);
      uint32_t g = 0, kv_item = 0, ucnt = 0;
      bool prev_valid = false, prev_first = false;
      uint32_t prev_g = 0, prev_vi = 0, prev_ucnt = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t pg, uint32_t vi, bool first, uint32_t pu) -> bool {
        if (!ptx::mbar_wait(&sh.p_full[pg & 1], (pg >> 1) & 1, abort, status, kStatusTimeout)) return false;
        if (first && pu > 0 && !ptx::mbar_wait(&sh.o_free, (pu - 1) & 1, abort, status, kStatusTimeout)) return false;
        const int s = vi % C::NSLOT;
        if (!ptx::mbar_wait(&sh.kv_full[s], (vi / C::NSLOT) & 1, abort, status, kStatusTimeout)) return false;
        ptx::tc_fence_after();
        const uint32_t pa = tS + (pg & 1) * 128;
        const uint32_t vb = kv_base + s * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          ptx::umma_ts(tO, pa + kk * 8, ptx::sw128_desc(vb + kk * 16 * 128, C::BLK, 1024), C::IDESC_O,
                       (kk > 0 || !first) ? 1u : 0u);
        ptx::umma_commit(&sh.pv_done[pg & 1]);
        ptx::umma_commit(&sh.kv_empty[s]);
        return true;
      };
      for (uint32_t ring = 0; ok; ++ring) {
        const int slot = ring & 1;
        if (!ptx::mbar_wait(&sh.unit_full[slot], (ring >> 1) & 1, abort, status, kStatusTimeout)) { ok = false; break; }
        const int32_t ntiles = sh.unit[slot][U_NTILES];
        ptx::mbar_arrive(&sh.unit_empty[slot]);
        if (ntiles < 0) break;
        const int qb = ucnt & 1;
        if (!ptx::mbar_wait(&sh.q_full[qb], (ucnt >> 1) & 1, abort, status, kStatusTimeout)) { ok = false; break; }
        const uint32_t qa = q_base + qb * C::Q_BYTES;
        for (int32_t t = 0; t < ntiles; ++t) {
          const uint32_t ki = kv_item, vi = kv_item + 1;
          kv_item += 2;
          const int s = ki % C::NSLOT;
          if (!ptx::mbar_wait(&sh.kv_full[s], (ki / C::NSLOT) & 1, abort, status, kStatusTimeout)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t kb = kv_base + s * C::TILE_BYTES;
          const uint32_t sd = tS + (g & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
            ptx::umma_ss(sd, ptx::sw128_desc(qa + off, 16, 1024), ptx::sw128_desc(kb + off, 16, 1024), C::IDESC_S,
                         kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(&sh.s_full[g & 1]);
          ptx::umma_commit(&sh.kv_empty[s]);
          if (t == ntiles - 1) ptx::umma_commit(&sh.q_empty[qb]);
          if (prev_valid && !issue_pv(prev_g, prev_vi, prev_first, prev_ucnt)) { ok = false; break; }
          prev_valid = true;
          prev_g = g;
          prev_vi = vi;
          prev_first = (t == 0);
          prev_ucnt = ucnt;
          ++g;
        }
        ++ucnt;
      }
      if (ok && prev_valid) issue_pv(prev_g, prev_vi, prev_first, prev_ucnt);
      // Drain: every MMA this CTA issued has completed before tensor memory is released.
      ptx::umma_commit(&sh.mma_drain);
      ptx::mbar_wait(&sh.mma_drain, 0, abort, status, kStatusTimeout);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------------- softmax warps 2..5
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0, pv_seen0 = 0, pv_seen1 = 0;
    bool ok = true;
    // The tcgen05.ld/st below are warp-collective, so every wait's outcome is made warp-uniform.
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kStatusTimeout));
    };
    // Waits until PV number k has completed. Completions of pv_done[k & 1] are observed strictly in
    // order, and at most one of them is ever pending when this runs, so parity tracking is exact.
    auto wait_pv = [&](uint32_t k) -> bool {
      uint32_t& seen = (k & 1) ? pv_seen1 : pv_seen0;
      while (seen <= (k >> 1)) {
        if (!wwait(&sh.pv_done[k & 1], seen & 1)) return false;
        ++seen;
      }
      return true;
    };
    for (uint32_t ring = 0; ok; ++ring) {
      const int slot = ring & 1;
      if (!wwait(&sh.unit_full[slot], (ring >> 1) & 1)) break;
      int32_t u[U_NFIELDS];
#pragma unroll
      for (int i = 0; i < U_NFIELDS; ++i) u[i] = sh.unit[slot][i];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
      const int32_t ntiles = u[U_NTILES];
      if (ntiles < 0) break;
      const int32_t pslot = row >> p.log2_group;
      const bool valid_row = pslot < u[U_NPOS];
      const int32_t i_pos = u[U_POS0] + (valid_row ? pslot : u[U_NPOS] - 1);
      const int32_t head = u[U_KVH] * G + (row & (G - 1));
      const bool is_global = u[U_GLOBAL] != 0;
      const int32_t S = u[U_SINK], W = u[U_WIN];
      const int32_t npages = u[U_AN] + u[U_BN];
      float m_run = -INFINITY, l_run = 0.f;

      for (int32_t t = 0; t < ntiles; ++t, ++g) {
        if (!wwait(&sh.s_full[g & 1], (g >> 1) & 1)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t sbuf = tS + (g & 1) * 128 + lane_off;
        float s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(sbuf + c * 32, reinterpret_cast<uint32_t*>(s) + c * 32);
        ptx::tmem_ld_wait();

        // Logical page of every slot of this tile; a row needs per-column bounds only if some key of
        // the tile is invisible to it (causal edge, window edge, sink tail, or a short last tile).
        int32_t lp[C::PPT];
        bool need_mask = false;
#pragma unroll
        for (int c = 0; c < C::PPT; ++c) {
          const int32_t x = t * C::PPT + c;
          if (x < npages) {
            lp[c] = unit_logical_page(u, unit_table_index(u, x));
            const int32_t j0 = lp[c] * P, j1 = j0 + P - 1;
            const bool all_vis = (j1 <= i_pos) && (is_global || j1 < S || j0 > i_pos - W);
            need_mask |= !all_vis;
          } else {
            lp[c] = -1;
            need_mask = true;
          }
        }
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < C::PPT; ++c) {
#pragma unroll
            for (int r = 0; r < P; ++r) {
              const int32_t j = lp[c] * P + r;
              const bool vis = lp[c] >= 0 && j <= i_pos && (is_global || j < S || j > i_pos - W);
              if (!vis) s[c * P + r] = -INFINITY;
            }
          }
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
        const float m_tile = mx * sl2;

        if (g >= 2 && !wait_pv(g - 2)) { ok = false; break; }
        const float m_new = fmaxf(m_run, m_tile);
        bool resc = false;
        if (t == 0) {
          m_run = m_new;
        } else {
          resc = m_new > m_run + 8.0f;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // O must hold every PV issued so far before it is rescaled in place.
          if (!wait_pv(g - 1)) { ok = false; break; }
          ptx::tc_fence_after();
          const float alpha = resc ? ptx::ex2(m_run - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(tO + lane_off + c * 32, r);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            ptx::tmem_st32(tO + lane_off + c * 32, r);
          }
          ptx::tmem_st_wait();
          if (resc) {
            l_run *= alpha;
            m_run = m_new;
          }
        }
        const float mu = (m_run == -INFINITY) ? 0.f : m_run;
        float rs = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ptx::ex2(fmaf(s[2 * c], sl2, -mu));
          const float p1 = ptx::ex2(fmaf(s[2 * c + 1], sl2, -mu));
          rs += p0 + p1;
          pk[c] = ptx::pack_bf16x2(p0, p1);
        }
        l_run += rs;
        ptx::tmem_st32(sbuf, pk);
        ptx::tmem_st32(sbuf + 32, pk + 32);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.p_full[g & 1]);
      }
      if (!ok) break;

      // ------------------------------------------------------------------------------ epilogue
      if (!wait_pv(g - 1)) break;
      ptx::tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int64_t qrow = (int64_t)u[U_QROW] + pslot;
      __nv_bfloat16* orow = p.o + (qrow * p.num_q_heads + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tO + lane_off + c * 32, r);
        ptx::tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          w[k] = ptx::pack_bf16x2(__uint_as_float(r[2 * k]) * inv_l, __uint_as_float(r[2 * k + 1]) * inv_l);
        if (valid_row) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      if (valid_row) p.lse[(int64_t)head * p.total_q + qrow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.o_free);
    }
  }

  // ------------------------------------------------------------------------------------ teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace segpaged
