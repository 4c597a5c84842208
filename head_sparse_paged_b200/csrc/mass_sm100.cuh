// mass_sm100.cuh -- attention mass each query-range token receives in a prefill, on B200 (sm_100a).
//
// The sparse FFN keeps the dense FFN for the top-k tokens by attention score (shshi.cn, "RedKnot技术原理"
// 3 "稀疏FFN动态调度"; bjdmk.com.cn, 二 item 2). The score read here is the mass a token receives:
//   mass[r] = sum_h sum_i exp(s_hij - LSE_hi) over query rows i whose visible set V_h(i) holds j,
// j the position of query row r. The row normalisers LSE come from the prefill, so this is a second
// pass over the (query tile, key tile) pairs whose keys lie in the query range -- a small share of the
// prefill's pairs when Lq << L.
//
// Work item: (sequence, KV head, 128-key tile x of the query range) and the query tiles that can see
// it. Logits are computed transposed, S^T = K Q^T (tcgen05.mma, M = 128 keys, N = 128 query rows,
// both operands K-major in 128B-swizzled shared memory, f32 in TMEM), so each thread of the mass
// warpgroup owns one key's TMEM lane and sums its row: no cross-thread reduction. The sum of an item
// goes to a per-(warpgroup, KV head, query row) partial; mass_reduce_kernel adds them in a fixed order.
//
// Per CTA, 14 warps:
//   warps 0-11 three mass warpgroups, taking the item's query tiles in turn (tile number mod 3 picks the
//              warpgroup and its TMEM buffer), so two exponentiate while the third waits on its logits:
//              tcgen05.ld of the key's 128 logits, exp2(s * scale * log2 e - LSE_i * log2 e) with
//              per-element bounds only on edge pairs, running sum in packed f32x2.
//   warp 12    producer: claims items, TMA-loads the key tile's pages once and every query tile
//              (same map as the prefill), and gathers the 128 rows' -LSE * log2 e into shared memory
//              (+inf LSE for rows past the query range, so they contribute exp2(-inf) = 0). Once the key
//              tile has landed it re-aligns its rows with the prefill's gather-time RoPE fragments, if
//              any, and releases it to the MMA warp.
//   warp 13    MMA issuer (whole warp, one elected lane issues): S^T into one of three TMEM buffers.
// Every wait is bounded, as in the prefill kernel.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"
#include "rope.cuh"
#include "sm100_ptx.cuh"

namespace segpaged {

// Fields of a mass work item (segpaged_mass_item::v).
enum MassField : int {
  M_SEQ = 0,   // sequence b
  M_KVH,       // KV head
  M_TILE,      // logical key tile x: keys [128 x, 128 x + 128)
  M_TOFF,      // offset of the (b, KV head) page-table entries
  M_NSINK,     // stored sink pages (storage_split)
  M_W0,        // first stored window page
  M_GLOBAL,    // head class
  M_SINK,
  M_WIN,
  M_Q0,        // first query position L - Lq
  M_L,         // context length
  M_QROW0,     // global row of the sequence's first query
  M_T0,        // first query tile (of 128/G positions) that can see the key tile
  M_NT,        // number of query tiles; -1 marks the end of the schedule
  M_TOTAL,     // stored pages of the (b, KV head)
  M_LQ,        // query positions of the sequence
  M_NFIELDS
};

constexpr int kMassWarpgroups = 3;          // warpgroups exponentiating, one TMEM buffer each
constexpr int kMassThreads = 32 * (4 * kMassWarpgroups + 2);
constexpr int32_t kMassStatusPageId = 1;
constexpr int32_t kMassStatusTimeout = 4;
constexpr int32_t kMassStatusUnit = 8;

template <int D, int P>
struct MassCfg {
  static constexpr int NH = D / 64;                   // 128-byte swizzle column blocks across D
  static constexpr int BLK = 128 * 128;               // bytes of one 64-column block of a 128-row tile
  static constexpr int TILE_BYTES = 128 * D * 2;      // key tile or query tile
  static constexpr int NWG = kMassWarpgroups;
  static constexpr int NQ = 5;                        // query-tile ring
  static constexpr int PPT = 128 / P;                 // pages per key tile
  static constexpr int SMEM_BYTES = TILE_BYTES * (1 + NQ) + NQ * 128 * 4 + 1024;
  static constexpr int THREADS = kMassThreads;
  static constexpr int PRODUCER = 4 * NWG, MMA = 4 * NWG + 1;   // warp roles after the mass warpgroups
  static constexpr uint32_t TMEM_COLS = NWG <= 2 ? 256 : 512;   // NWG S^T buffers of 128 columns
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(128, 128, 0, 0);
};

struct MassParams {
  const int32_t* page_table;
  int64_t page_table_len;
  const int32_t* items;  // [num_items][M_NFIELDS]
  int32_t num_items;
  int32_t* counter;      // zeroed before the launch
  int32_t* status;       // nullable
  const float* lse;      // [Hq, total_q], natural log
  float* part;           // [2 warpgroups][Hkv][total_q]
  int32_t total_q, num_q_heads, num_kv_heads, num_pages, log2_group;
  float scale_log2;      // softmax_scale * log2(e)
  RopeFragments frags;   // offs == nullptr: keys are used as stored
};

struct MassShared {
  uint64_t item_full[2], item_empty[2];
  uint64_t k_full, k_ready, k_empty;
  uint64_t q_full[8], q_empty[8];
  uint64_t s_full[4], s_empty[4];
  uint64_t drain;
  __align__(16) int32_t item[2][M_NFIELDS];
  uint32_t tmem_base;
  int abort;
};

template <int D, int P>
__global__ void __launch_bounds__(kMassThreads, 1)
    segpaged_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const MassParams p) {
  using C = MassCfg<D, P>;
  static_assert(C::NQ <= 8 && C::NWG <= 4, "barrier arrays hold eight query slots and four buffers");
  extern __shared__ uint8_t smem_raw[];
  __shared__ MassShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                                   // key tile
  uint8_t* sQ = smem + C::TILE_BYTES;                   // NQ query tiles
  float* s_nlse = reinterpret_cast<float*>(smem + C::TILE_BYTES * (1 + C::NQ));   // [NQ][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sh.abort;
  int32_t* status = p.status;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.item_full[i], 1);
      ptx::mbar_init(&sh.item_empty[i], 1 + 4 * C::NWG);   // MMA warp + every mass warp
    }
    for (int i = 0; i < C::NWG; ++i) {
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.s_empty[i], 4);      // the 4 warps of the buffer's warpgroup
    }
    for (int i = 0; i < C::NQ; ++i) {
      ptx::mbar_init(&sh.q_full[i], 1);
      ptx::mbar_init(&sh.q_empty[i], 5);      // MMA commit + the 4 warps that read the tile's LSE
    }
    ptx::mbar_init(&sh.k_full, 1);
    ptx::mbar_init(&sh.k_ready, 1);
    ptx::mbar_init(&sh.k_empty, 1);
    ptx::mbar_init(&sh.drain, 1);
    sh.abort = 0;
    ptx::mbar_fence_init();
  }
  if (warp == C::PRODUCER && lane == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_k);
  }
  if (warp == C::MMA) {
    ptx::tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // The key tile starts zeroed: pages a tile skips (keys before the query range) keep finite data.
  for (int x = threadIdx.x; x < C::TILE_BYTES / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(sK)[x] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int G = 1 << p.log2_group;
  const int npos = 128 >> p.log2_group;

  if (warp == C::PRODUCER) {
    // ------------------------------------------------------------------------------ producer
    uint32_t qi = 0, q_issued = 0;
    int32_t k_ring = -1;
    for (uint32_t ring = 0;; ++ring) {
      const int slot = ring & 1;
      int go = 1;
      if (lane == 0) go = ptx::mbar_wait(&sh.item_empty[slot], ((ring >> 1) & 1) ^ 1, abort, status, kMassStatusTimeout);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      int32_t u = 0;
      if (lane == 0) u = atomicAdd(p.counter, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      const bool done = u >= p.num_items;
      int32_t* I = sh.item[slot];
      if (done) {
        if (lane == 0) I[M_NT] = -1;
      } else if (lane < M_NFIELDS / 4) {
        reinterpret_cast<int4*>(I)[lane] = reinterpret_cast<const int4*>(p.items + (int64_t)u * M_NFIELDS)[lane];
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.item_full[slot]);
      if (done) break;
      const int32_t x = I[M_TILE], q0 = I[M_Q0], L = I[M_L], kvh = I[M_KVH], qrow0 = I[M_QROW0];
      const int32_t t0 = I[M_T0], nt = I[M_NT], Lq = I[M_LQ];
      // key tile: the pages holding a key of the query range
      if (lane == 0) {
        go = ptx::mbar_wait(&sh.k_empty, (ring & 1) ^ 1, abort, status, kMassStatusTimeout);
        if (go) {
          int32_t pid[C::PPT];
          int32_t n_ok = 0;
#pragma unroll
          for (int c = 0; c < C::PPT; ++c) {
            const int32_t lp = x * C::PPT + c;
            pid[c] = -1;
            if ((int64_t)lp * P + P <= q0 || (int64_t)lp * P >= L) continue;
            const int32_t idx = I[M_GLOBAL] ? lp : (lp < I[M_NSINK] ? lp : I[M_NSINK] + (lp - I[M_W0]));
            if (idx < 0 || idx >= I[M_TOTAL] || (int64_t)I[M_TOFF] + idx >= p.page_table_len) {
              if (status) atomicOr(status, kMassStatusUnit);
              continue;
            }
            int32_t v = p.page_table[(int64_t)I[M_TOFF] + idx];
            if (v < 0 || v >= p.num_pages) {
              if (status) atomicOr(status, kMassStatusPageId);
              v = 0;
            }
            pid[c] = v;
            ++n_ok;
          }
          ptx::mbar_arrive_expect_tx(&sh.k_full, (uint32_t)(n_ok * P * D * 2));
#pragma unroll
          for (int c = 0; c < C::PPT; ++c) {
            if (pid[c] < 0) continue;
#pragma unroll
            for (int h = 0; h < C::NH; ++h)
              ptx::tma_load_3d(sK + h * C::BLK + c * P * 128, &tm_k, h * 64, 0, pid[c], &sh.k_full);
          }
          k_ring = (int32_t)ring;
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      // query tiles with their rows' -LSE * log2(e); the values of the next tile are loaded while the
      // current one waits for its slot and is issued, so the gather's latency stays off the critical path
      auto gather = [&](int32_t t, float (&nl)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = lane + 32 * k;
          const int32_t posl = t * npos + (c >> p.log2_group);
          nl[k] = -INFINITY;
          if (posl < Lq && qrow0 + posl < p.total_q) {
            const int32_t head = kvh * G + (c & (G - 1));
            nl[k] = -p.lse[(int64_t)head * p.total_q + qrow0 + posl] * 1.4426950408889634f;
          }
        }
      };
      float cur[4];
      gather(t0, cur);
      for (int32_t t = t0; t < t0 + nt; ++t, ++qi) {
        const int s = qi % C::NQ;
        float nxt[4] = {0.f, 0.f, 0.f, 0.f};
        if (t + 1 < t0 + nt) gather(t + 1, nxt);
        if (lane == 0) go = ptx::mbar_wait(&sh.q_empty[s], ((qi / C::NQ) & 1) ^ 1, abort, status, kMassStatusTimeout);
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          s_nlse[s * 128 + lane + 32 * k] = cur[k];
          cur[k] = nxt[k];
        }
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&sh.q_full[s], C::TILE_BYTES);
#pragma unroll
          for (int h = 0; h < C::NH; ++h)
            ptx::tma_load_3d(sQ + s * C::TILE_BYTES + h * C::BLK, &tm_q, h * 64, kvh * G, qrow0 + t * npos,
                             &sh.q_full[s]);
          q_issued = qi + 1;
        }
        if (t == t0) {
          // the key tile: wait until it has landed, re-align its fragment rows, release it to the MMA warp
          if (lane == 0) go = ptx::mbar_wait(&sh.k_full, ring & 1, abort, status, kMassStatusTimeout);
          if (!__shfl_sync(0xffffffffu, go, 0)) break;
          if (p.frags.offs) {
            const int32_t flo = p.frags.offs[I[M_SEQ]], fhi = p.frags.offs[I[M_SEQ] + 1];
            if (fhi > flo) {
              constexpr int CH = D / 16;
              for (int xx = lane; xx < 128 * CH; xx += 32) {
                const int r = xx / CH, c = xx % CH;
                const int32_t f = rope_fragment_of(p.frags.start, flo, fhi, x * 128 + r);
                if (f >= 0) rope_rotate_smem_chunk<D>(sK, r, c, p.frags.cs + (int64_t)f * D);
              }
              ptx::fence_proxy_async_smem();
            }
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.k_ready);
        }
      }
      if (!go) break;
    }
    // After giving up, wait (bounded, ignoring the abort flag) for this warp's copies in flight.
    if (lane == 0 && *abort) {
      if (k_ring >= 0) ptx::mbar_wait(&sh.k_full, (uint32_t)k_ring & 1, nullptr, status, kMassStatusTimeout);
      const uint32_t first = q_issued > (uint32_t)C::NQ ? q_issued - C::NQ : 0u;
      for (uint32_t it = first; it < q_issued; ++it)
        ptx::mbar_wait(&sh.q_full[it % C::NQ], (it / C::NQ) & 1, nullptr, status, kMassStatusTimeout);
    }
    __syncwarp();
  } else if (warp == C::MMA) {
    // --------------------------------------------------------------------------- MMA issuer
    const uint32_t leader = ptx::elect_one();
    const uint32_t k_base = ptx::smem_addr(sK), q_base = ptx::smem_addr(sQ);
    const uint64_t kdesc = ptx::sw128_desc(k_base, 16, 1024);
    uint32_t qi = 0, si = 0;
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kMassStatusTimeout));
    };
    bool ok = true;
    for (uint32_t ring = 0; ok; ++ring) {
      const int slot = ring & 1;
      if (!wait(&sh.item_full[slot], (ring >> 1) & 1)) break;
      const int32_t nt = sh.item[slot][M_NT];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.item_empty[slot]);
      if (nt < 0) break;
      if (!wait(&sh.k_ready, ring & 1)) break;
      for (int32_t t = 0; t < nt; ++t, ++qi, ++si) {
        const int s = qi % C::NQ, b = si % C::NWG;
        if (!wait(&sh.q_full[s], (qi / C::NQ) & 1) || !wait(&sh.s_empty[b], ((si / C::NWG) & 1) ^ 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t qdesc = ptx::sw128_desc(q_base + s * C::TILE_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * C::BLK + (kk & 3) * 32) >> 4);
          ptx::umma_ss(leader, tmem + b * 128, kdesc + off, qdesc + off, C::IDESC, kk > 0 ? 1u : 0u);
        }
        ptx::umma_commit(leader, &sh.s_full[b]);
        ptx::umma_commit(leader, &sh.q_empty[s]);
      }
      if (!ok) break;
      ptx::umma_commit(leader, &sh.k_empty);
    }
    __syncwarp();
    ptx::umma_commit(leader, &sh.drain);
    ptx::mbar_wait(&sh.drain, 0, nullptr, status, kMassStatusTimeout);
    __syncwarp();
  } else {
    // ----------------------------------------------------------------------- mass warpgroups
    const int wg = warp >> 2;                            // takes the tiles g with g % NWG == wg
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                 // key row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint64_t sl2_2 = f2_pack(p.scale_log2, p.scale_log2);
    uint32_t qi = 0, si = 0;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kMassStatusTimeout));
    };
    for (uint32_t ring = 0;; ++ring) {
      const int slot = ring & 1;
      if (!wwait(&sh.item_full[slot], (ring >> 1) & 1)) break;
      const int32_t* I = sh.item[slot];
      const int32_t nt = I[M_NT];
      if (nt < 0) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.item_empty[slot]);
        break;
      }
      const int32_t j = I[M_TILE] * 128 + row;           // this thread's key position
      const int32_t q0 = I[M_Q0], t0 = I[M_T0];
      const bool is_global = I[M_GLOBAL] != 0;
      const int32_t S = I[M_SINK], W = I[M_WIN];
      float sum = 0.f;
      bool ok = true;
      for (int32_t t = 0; t < nt; ++t, ++qi, ++si) {
        const int s = qi % C::NQ, b = si % C::NWG;
        if (b != wg) continue;
        // The query tile's positions [pa, pb] and which of them see key j, worked out before the logits are
        // ready: positions j .. j + W - 1 for a key of a local head past its sink, j .. pb otherwise. As tile
        // columns (G per position) that is one range, kept as bits for the edge pairs.
        const int32_t pa = q0 + (t0 + t) * npos, pb = pa + npos - 1;
        const bool none = j > pb || (!is_global && j >= S && j <= pa - W);
        const bool all = j <= pa && (is_global || j < S || j > pb - W);
        const int32_t vlo = max(j, pa);
        const int32_t vhi = (is_global || j < S || W > pb - j) ? pb : j + W - 1;
        const int32_t clo = (vlo - pa) * G, chi = (vhi - pa + 1) * G;     // chi < clo: nothing visible
        if (!wwait(&sh.s_full[b], (si / C::NWG) & 1) || !wwait(&sh.q_full[s], (qi / C::NQ) & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const float* nl = s_nlse + s * 128;
        const uint32_t sbuf = tmem + b * 128 + lane_off;
        uint64_t acc[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        // the key's 128 logits in two halves of 64 columns (fewer live registers); the buffer is released
        // once the second half is in registers
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float v[64];
          ptx::tmem_ld32(sbuf + half * 64, reinterpret_cast<uint32_t*>(v));
          ptx::tmem_ld32(sbuf + half * 64 + 32, reinterpret_cast<uint32_t*>(v) + 32);
          ptx::tmem_ld_wait();
          if (half == 1) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sh.s_empty[b]);
          }
          if (none) continue;
          if (!all) {
            // edge pair: logits of rows that cannot see key j drop out (masked before the exponentials,
            // so the exponential loop below has no per-element branch)
            const uint32_t mw[2] = {range_bits(clo - half * 64, chi - half * 64),
                                    range_bits(clo - half * 64 - 32, chi - half * 64 - 32)};
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (!((mw[c >> 5] >> (c & 31)) & 1u)) v[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 n4 = *reinterpret_cast<const float4*>(nl + half * 64 + c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e = c + 2 * h;
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(v[e], v[e + 1]), sl2_2, h ? f2_pack(n4.z, n4.w) : f2_pack(n4.x, n4.y)), x0, x1);
              acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(ptx::ex2(x0), ptx::ex2(x1)));
            }
          }
        }
        if (!none) {
          float t0f, t1f;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), t0f, t1f);
          sum += t0f + t1f;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.q_empty[s]);
      }
      if (!ok) break;
      if (j >= q0 && j < I[M_L]) {
        const int64_t r = (int64_t)I[M_QROW0] + (j - q0);
        if (I[M_KVH] >= 0 && I[M_KVH] < p.num_kv_heads && r < p.total_q)
          p.part[((int64_t)wg * p.num_kv_heads + I[M_KVH]) * p.total_q + r] = sum;
        else if (status) atomicOr(status, kMassStatusUnit);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.item_empty[slot]);
    }
  }

  // every warp arrives at the block barrier converged, so each is counted once before tensor memory is freed
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::MMA) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// mass[r] = sum over planes k (warpgroup-major, then KV head, in order) of part[k][r].
__global__ void mass_reduce_kernel(const float* __restrict__ part, float* __restrict__ mass, int32_t total_q,
                                   int32_t num_planes) {
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < total_q; r += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < num_planes; ++k) s += part[(int64_t)k * total_q + r];
    mass[r] = s;
  }
}

}  // namespace segpaged
