// prefill_sm100.cuh -- EXECUTE: SegPagedAttention prefill on B200 (sm_100a).
//
// One persistent kernel runs every query head over exactly its own ragged, paged KV with no mask
// tensor (zhichai.net, 事件内容 item 3; bjdmk.com.cn, 二 item 3; aiboss88.com, 技術原則, item on paged
// storage removing the attn_mask penalty). Visibility: key j is visible to query position i iff
// j <= i and (global head, or j < S, or j > i - W).
//
// Work: units of (sequence, KV head, up to 2 x 128/G query positions x G query heads), planned on the
// host with their visible page ranges and sorted longest-first; CTAs (one per SM) claim them through a
// global atomic counter. A unit is two 128-row query tiles that share every K/V tile of the unit.
//
// Per CTA, 12 warps (3 warpgroups):
//   warps 0-3   softmax for query tile 0, warps 4-7 softmax for query tile 1: one tile row per thread.
//               tcgen05.ld of the S row, per-row bounds only on edge tiles, row max (3-input max),
//               lazy O rescale (only when the running max grows by more than 2^8), exp2 on the MUFU
//               unit (one pair in eight on the FMA pipe by a cubic, beside it), row sum and scaling in packed
//               f32x2 arithmetic, P written back to TMEM as bf16 over
//               S and published in two halves of 64 keys, and the epilogue (O / l -> bf16,
//               LSE = ln 2 * (m + log2 l)).
//   warp 8      producer (whole warp: page-table lookups; lane 0: barriers and TMA): claims units, TMA-loads both Q tiles (3-D map over [rows, Hq, D], box
//               64 x G x 128/G) and, for every 128-key tile, the K and V pages (3-D map over
//               [pages, P, D], coordinate = physical page id) into 128B-swizzled shared-memory slots.
//   warp 9      MMA issuer (whole warp, one elected lane issues), in the order PV0(j-1), S0(j), PV1(j-1), S1(j): S_t = Q_t K^T
//               (tcgen05.mma, both operands in shared memory, f32 in TMEM) and O_t += P_t V (P from
//               TMEM, V MN-major from shared memory; keys 0-63 as soon as that half of P is written).
//               The commit that publishes S_t(j) also covers PV_t(j-1), so when a softmax warp sees
//               S_t(j) its O_t is stable and can be rescaled.
//   warps 10-11 idle, or when appending (fused append-and-attend) writing the new keys and values of the
//               unit's query positions into their pool pages.
//   warps 12-15 only with ROPE: the gather-time RoPE re-alignment. They rotate each K tile in shared
//               memory once it lands (keys of reused fragments, from their original to their actual
//               positions, per sequence fragment) and only then release it to the MMA warp.
// Every wait is bounded: on a timeout the CTA raises its abort flag, reports SEGPAGED_STATUS_TIMEOUT,
// waits (bounded) for its TMA copies and MMAs in flight, and frees its tensor memory before returning.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "combine_kernel.cuh"
#include "plan.h"
#include "rope.cuh"
#include "sm100_ptx.cuh"

namespace segpaged {

constexpr int32_t kStatusPageId = 1;
constexpr int32_t kStatusTimeout = 4;
constexpr int32_t kStatusUnit = 8;

template <int D, int P, bool ROPE = false>
struct PrefillCfg {
  static constexpr int BM = 128;                 // rows of one query tile (positions x heads)
  static constexpr int BN = 128;                 // keys per KV tile
  static constexpr int NH = D / 64;              // 128-byte swizzle column blocks across D
  static constexpr int BLK = BN * 128;           // bytes of one 64-column block of a 128-row tile
  static constexpr int TILE_BYTES = BN * D * 2;  // one K or V tile
  static constexpr int Q_BYTES = BM * D * 2;     // one query tile
  static constexpr int NSLOT = (D == 128) ? 5 : 10;
  static constexpr int PPT = BN / P;             // pages per KV tile
  static constexpr int SMEM_BYTES = 2 * Q_BYTES + NSLOT * TILE_BYTES + 1024;
  static constexpr int THREADS = ROPE ? 512 : 384;   // ROPE: a fourth warpgroup rotates K tiles
  static constexpr uint32_t TMEM_COLS = 512;     // S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D)
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t IDESC_O = ptx::idesc_bf16_f32(128, D, 0, 1);
  // Register split (setmaxnreg): 256 softmax threads x 208 + 128 other threads x 80 = 63488, within the
  // 384 x 168 = 64512 registers the block is launched with; with ROPE 256 x 192 + 128 x 64 (producer,
  // MMA) + 128 x 64 (RoPE warpgroup) = 65536 = 512 x 128.
  static constexpr int REGS_SOFTMAX = ROPE ? 192 : 208;
  static constexpr int REGS_OTHER = ROPE ? 64 : 80;
  static constexpr int REGS_ROPE = 64;
  static constexpr int LAUNCH_REGS = ROPE ? 128 : 168;
  static_assert(256 * REGS_SOFTMAX + 128 * REGS_OTHER + (ROPE ? 128 * REGS_ROPE : 0) <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch budget");
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
  float* part_o;         // [partial slots][D/4][256 rows] fp32 4-column groups (partial_o_index): O / l of one
                         // chunk of a split unit
  float* part_lse;       // [partial slots][256 rows] fp32: LSE of that chunk (natural log)
  int32_t total_q, num_q_heads, num_pages, log2_group;
  int32_t num_partials;  // partial slots in part_o / part_lse
  int32_t num_seqs;      // sequences of the call (RoPE: entries of frags.offs minus one)
  float scale_log2;      // softmax_scale * log2(e)
  RopeFragments frags;   // used by the ROPE variant only
  // fused append-and-attend: the new keys/values [total_q, Hkv, D] are read for the new-page tiles and
  // written into their pool pages by warps 10-11
  int32_t append;
  int32_t num_kv_heads;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
};

constexpr int kRopeSmemFragments = 64;    // fragment starts of a sequence cached in shared memory

template <bool ROPE>
struct PrefillShared {
  uint64_t unit_full[2], unit_empty[2];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_half[2], p_full[2], o_full[2], o_free[2];
  uint64_t mma_drain;
  uint64_t kv_full[11], kv_empty[11];
  uint64_t k_rot[11];      // ROPE: K tile of tile count n rotated (ring over n % NSLOT), ready for the MMA
  __align__(16) int32_t unit[2][U_NFIELDS];
  int32_t frag_start[ROPE ? kRopeSmemFragments : 1];   // ROPE: the current unit's sequence fragment starts
  float ml[256];              // shared half units: warpgroup 1's running max and sum per row, for the merge
  uint64_t ml_full, ml_empty; // ... written by warpgroup 1 (4 warps), read by warpgroup 0 (4 warps)
  uint32_t tmem_base;
  int abort;
};

// One pair of exponentials in every kExpCubicEvery runs on the FMA and integer pipes instead of MUFU (0: none).
constexpr int kExpCubicEvery = 8;

// List position x of a unit -> page-table index.
__device__ __forceinline__ int32_t unit_table_index(const int32_t* u, int32_t x) {
  return x < u[U_AN] ? x : u[U_B0] + (x - u[U_AN]);
}
// Page-table index -> logical page.
__device__ __forceinline__ int32_t unit_logical_page(const int32_t* u, int32_t idx) {
  return idx < u[U_NSINK] ? idx : u[U_W0] + (idx - u[U_NSINK]);
}

// Kernel variants: the plain prefill, gather-time RoPE, and fused append-and-attend.
constexpr int kModePlain = 0, kModeRope = 1, kModeAppend = 2;

// HALF (chosen per launch): 0 -- every unit has rows in both query tiles; 1 -- the plan has half units;
// 2 -- every unit is a half unit.
template <int D, int P, int MODE, int HALF>
__global__ void __launch_bounds__(MODE == kModeRope ? 512 : 384, 1)
    segpaged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kn,
                            const __grid_constant__ CUtensorMap tm_vn, const PrefillParams p) {
  constexpr bool ROPE = MODE == kModeRope, APPEND = MODE == kModeAppend;
  // SHARED_HALF (the plan has half units): a unit with rows in one query tile only still keeps both softmax
  // warpgroups busy -- its KV tiles alternate between them (S buffer, P, O accumulator t = tile & 1) and
  // warpgroup 0 merges the two accumulators at the end. The variant without it keeps the long-unit path
  // free of the extra bookkeeping (about 3 % on long layers).
  // ALL_HALF (every unit is a half unit -- short query ranges, decode-like batches): the second query
  // buffer is never loaded, so it becomes one more K/V slot; these launches stream pages and are bound by
  // how many loads each SM keeps in flight.
  constexpr bool SHARED_HALF = HALF != 0, ALL_HALF = HALF == 2;
  using C = PrefillCfg<D, P, ROPE>;
  constexpr int NSLOT = C::NSLOT + (ALL_HALF ? 1 : 0);   // K/V slots of this variant
  static_assert(C::Q_BYTES == C::TILE_BYTES, "a query buffer doubles as a K/V slot");
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrefillShared<ROPE> sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                      // 2 query tiles x Q_BYTES (1 with ALL_HALF)
  uint8_t* sKV = smem + (ALL_HALF ? 1 : 2) * C::Q_BYTES;   // NSLOT x TILE_BYTES
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sh.abort;
  int32_t* status = p.status;

  // Physical page id of list position 32 * batch + lane of unit U (-1 past its list; 0, and a status bit, for a
  // table index or page id outside the call's arrays).
  auto fetch_pid = [&](const int32_t* U, int32_t batch) -> int32_t {
    const int32_t x = (batch << 5) + lane;
    const int64_t toff = U[U_TOFF];
    int32_t pid = -1;
    if (x < U[U_AN] + U[U_BN]) {
      const int32_t idx = unit_table_index(U, x);
      pid = 0;
      if (idx < 0 || idx >= U[U_TOTAL] || toff + idx < 0 || toff + idx >= p.page_table_len) {
        if (status) atomicOr(status, kStatusUnit);
      } else {
        pid = p.page_table[toff + idx];
        if (pid < 0 || pid >= p.num_pages) {
          if (status) atomicOr(status, kStatusPageId);
          pid = 0;
        }
      }
    }
    return pid;
  };
  // The producer's first unit is unit blockIdx.x (the grid never exceeds the unit count). Its descriptor and the
  // page ids of its first 32 list positions are fetched now, so those global-memory round trips overlap the
  // block's set-up instead of delaying the first query and K/V loads.
  int32_t pre_batch = -1, pre_pid = -1;
  if (warp == 8) {
    int32_t* U0 = sh.unit[0];
    if (lane < U_NFIELDS / 4)
      reinterpret_cast<int4*>(U0)[lane] = reinterpret_cast<const int4*>(p.units + (int64_t)blockIdx.x * U_NFIELDS)[lane];
    __syncwarp();
    pre_batch = (U0[U_T0] * C::PPT) >> 5;
    pre_pid = fetch_pid(U0, pre_batch);
  }

  // ---------------------------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&sh.unit_full[i], 1);
      // MMA warp + 8 softmax warps (+ 4 RoPE warps, or + 2 append warps)
      ptx::mbar_init(&sh.unit_empty[i], ROPE ? 13 : (APPEND ? 11 : 9));
      ptx::mbar_init(&sh.s_full[i], 1);
      ptx::mbar_init(&sh.p_half[i], 4);
      ptx::mbar_init(&sh.p_full[i], 4);
      ptx::mbar_init(&sh.o_full[i], 1);
      ptx::mbar_init(&sh.o_free[i], 4);
    }
    ptx::mbar_init(&sh.q_full, 1);
    ptx::mbar_init(&sh.q_empty, 1);
    ptx::mbar_init(&sh.mma_drain, 1);
    ptx::mbar_init(&sh.ml_full, 4);
    ptx::mbar_init(&sh.ml_empty, 4);
    for (int i = 0; i < NSLOT; ++i) {
      ptx::mbar_init(&sh.kv_full[i], 1);
      ptx::mbar_init(&sh.kv_empty[i], 1);
      ptx::mbar_init(&sh.k_rot[i], 4);
    }
    sh.abort = 0;
    ptx::mbar_fence_init();
  }
  if (warp == 8 && lane == 0) {
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
    if (APPEND) {
      ptx::tma_prefetch_desc(&tm_kn);
      ptx::tma_prefetch_desc(&tm_vn);
    }
  }
  if (warp == 9) {
    ptx::tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // KV slots start zeroed: a partial tile (pages smaller than a tile) leaves earlier (finite) data in the
  // rows it does not load, and those columns are masked. With one page per tile every used slot is loaded
  // whole, and the start-up saves the stores.
  if constexpr (C::PPT > 1) {
    for (int x = threadIdx.x; x < NSLOT * C::TILE_BYTES / 16; x += blockDim.x)
      reinterpret_cast<uint4*>(sKV)[x] = make_uint4(0, 0, 0, 0);
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int G = 1 << p.log2_group;
  const int npos = C::BM >> p.log2_group;    // positions per query tile

  if (warp >= 8) {
    if (warp < 12) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_ROPE));
    if (warp == 8) {
      // ---------------------------------------------------------------------------- producer
      // The whole warp walks the schedule; lane 0 does the barrier and TMA work, and the 32 lanes fetch
      // the page-table entries of 32 list positions at once, so a tile's loads never wait on a lookup.
      uint32_t kv_item = 0;
      uint32_t kv_issued = 0;        // lane 0: KV items whose loads were issued
      int32_t q_ring = -1;           // lane 0: ring index of the last query-tile load issued
      for (uint32_t ring = 0;; ++ring) {
        const int slot = ring & 1;
        int go = 1;
        if (lane == 0) go = ptx::mbar_wait(&sh.unit_empty[slot], ((ring >> 1) & 1) ^ 1, abort, status, kStatusTimeout);
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        // claim the next unit only once a ring slot is free, so no CTA sits on work it cannot start; the first
        // unit of CTA i is unit i (the grid never exceeds the unit count), which takes the atomic off the
        // start-up path, and later claims come from the counter, offset by the grid. A launch with one unit
        // per CTA never touches the counter (the host does not clear it for such a launch).
        int32_t u = 0;
        if (lane == 0)
          u = ring == 0 ? (int32_t)blockIdx.x
                        : ((int32_t)gridDim.x >= p.num_units ? p.num_units : (int32_t)gridDim.x + atomicAdd(p.counter, 1));
        u = __shfl_sync(0xffffffffu, u, 0);
        const bool done = u >= p.num_units;
        int32_t* U = sh.unit[slot];
        if (done) {
          if (lane == 0) U[U_NTILES] = -1;
        } else if (ring > 0 && lane < U_NFIELDS / 4) {    // ring 0: fetched before the set-up
          reinterpret_cast<int4*>(U)[lane] = reinterpret_cast<const int4*>(p.units + (int64_t)u * U_NFIELDS)[lane];
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_full[slot]);
        if (done) break;
        // both query tiles: the unit's positions [0, npos) and [npos, 2 npos)
        if (lane == 0) {
          go = ptx::mbar_wait(&sh.q_empty, (ring & 1) ^ 1, abort, status, kStatusTimeout);
          if (go) {
            // a half unit has no rows in its second query tile; with ALL_HALF a unit that is not half is a
            // plan that does not match the launch, and only its first query tile is computed
            if (ALL_HALF && !U[U_HALF] && status) atomicOr(status, kStatusUnit);
            const int nq = (ALL_HALF || U[U_HALF]) ? 1 : 2;
            ptx::mbar_arrive_expect_tx(&sh.q_full, nq * C::Q_BYTES);
            q_ring = (int32_t)ring;
            for (int t = 0; t < nq; ++t)
#pragma unroll
              for (int h = 0; h < C::NH; ++h)
                ptx::tma_load_3d(sQ + t * C::Q_BYTES + h * C::BLK, &tm_q, h * 64, U[U_KVH] * G,
                                 U[U_QROW] + t * npos, &sh.q_full);
          }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        const int32_t t0 = U[U_T0];
        const int32_t ntiles = U[U_NTILES];
        const int32_t noldt = U[U_NOLDT], new0 = U[U_NEW0], nnew = U[U_NNEW];
        const int32_t kvh = U[U_KVH], newrow0 = U[U_CUQ] - U[U_SPLITQ];   // new-K/V row of key position 0
        if (nnew > 0 && !APPEND && lane == 0 && status) atomicOr(status, kStatusUnit);   // append plan, plain call
        int32_t batch = ring == 0 ? pre_batch : -1;   // my_pid: page id of list position 32 * batch + lane
        int32_t my_pid = ring == 0 ? pre_pid : -1;
        int ok = 1;
        for (int32_t j = t0; j < t0 + ntiles && ok; ++j) {
          int32_t pages[C::PPT];             // physical page ids (pool tiles) or logical pages (new-page tiles)
          int32_t n_ok = 0;
          const bool fresh = APPEND && j >= noldt;
          if (!fresh) {
            const int32_t x0 = j * C::PPT;     // a tile's PPT positions never straddle a batch of 32
            if ((x0 >> 5) != batch) {
              batch = x0 >> 5;
              my_pid = fetch_pid(U, batch);
            }
#pragma unroll
            for (int c = 0; c < C::PPT; ++c) {
              pages[c] = __shfl_sync(0xffffffffu, my_pid, (x0 + c) & 31);
              n_ok += pages[c] >= 0 ? 1 : 0;
            }
          } else {
#pragma unroll
            for (int c = 0; c < C::PPT; ++c) {
              const int32_t xn = (j - noldt) * C::PPT + c;
              pages[c] = xn < nnew ? new0 + xn : -1;
              n_ok += pages[c] >= 0 ? 1 : 0;
            }
          }
          if (lane == 0) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {  // K then V
              const uint32_t item = kv_item + which;
              const int s = item % NSLOT;
              if (!ptx::mbar_wait(&sh.kv_empty[s], ((item / NSLOT) & 1) ^ 1, abort, status, kStatusTimeout)) {
                ok = 0;
                break;
              }
              ptx::mbar_arrive_expect_tx(&sh.kv_full[s], (uint32_t)(n_ok * P * D * 2));
              uint8_t* dst = sKV + s * C::TILE_BYTES;
#pragma unroll
              for (int c = 0; c < C::PPT; ++c) {
                if (pages[c] < 0) continue;
#pragma unroll
                for (int h = 0; h < C::NH; ++h) {
                  if (!fresh)
                    ptx::tma_load_3d(dst + h * C::BLK + c * P * 128, which ? &tm_v : &tm_k, h * 64, 0, pages[c],
                                     &sh.kv_full[s]);
                  else   // P rows of the new K/V from key position pages[c] * P (rows before q0 are masked)
                    ptx::tma_load_3d(dst + h * C::BLK + c * P * 128, which ? &tm_vn : &tm_kn, h * 64, kvh,
                                     newrow0 + pages[c] * P, &sh.kv_full[s]);
                }
              }
              kv_issued = item + 1;
            }
          }
          kv_item += 2;
          ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (!ok) break;
      }
      // After giving up, wait (bounded, ignoring the abort flag) for the copies this warp issued, so
      // none lands in shared memory after the CTA has exited.
      if (lane == 0 && *abort) {
        const uint32_t first = kv_issued > (uint32_t)NSLOT ? kv_issued - NSLOT : 0u;
        for (uint32_t it = first; it < kv_issued; ++it)
          ptx::mbar_wait(&sh.kv_full[it % NSLOT], (it / NSLOT) & 1, nullptr, status, kStatusTimeout);
        if (q_ring >= 0) ptx::mbar_wait(&sh.q_full, (uint32_t)q_ring & 1, nullptr, status, kStatusTimeout);
      }
      __syncwarp();
    } else if (warp == 9) {
      // -------------------------------------------------------------------------- MMA issuer
      // The whole warp walks the schedule, so barrier parities, slots and descriptors are warp-uniform
      // values; one elected lane issues each tcgen05.mma and tcgen05.commit.
      const uint32_t leader = ptx::elect_one();
      const uint32_t q_base = ptx::smem_addr(sQ), kv_base = ptx::smem_addr(sKV);
      uint32_t kv_item = 0, act[2] = {0, 0}, pcount[2] = {0, 0};
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kStatusTimeout));
      };
      // O_t (+)= P_t V for the V tile in KV item vi; `first` starts the unit's accumulation. The softmax
      // warps publish P_t in two halves of 64 keys: the first half's MMAs run while they finish the second.
      auto issue_pv = [&](int t, uint32_t vi, bool first, bool wait_v) -> bool {
        if (!wait(&sh.p_half[t], pcount[t] & 1)) return false;
        if (first && act[t] > 0 && !wait(&sh.o_free[t], (act[t] - 1) & 1)) return false;
        const int s = vi % NSLOT;
        if (wait_v && !wait(&sh.kv_full[s], (vi / NSLOT) & 1)) return false;
        ptx::tc_fence_after();
        const uint32_t pa = tmem + t * 128;                 // P_t: bf16 pairs over the first 64 columns of S_t
        const uint32_t od = tmem + 256 + t * D;
        const uint64_t vdesc = ptx::sw128_desc(kv_base + s * C::TILE_BYTES, C::BLK, 1024);
#pragma unroll
        for (int kk = 0; kk < C::BN / 32; ++kk)             // 16 keys = 2048 B of V = 128 in the address field
          ptx::umma_ts(leader, od, pa + kk * 8, vdesc + (uint64_t)(kk * 128), C::IDESC_O,
                       (kk > 0 || !first) ? 1u : 0u);
        if (!wait(&sh.p_full[t], pcount[t] & 1)) return false;
        ++pcount[t];
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = C::BN / 32; kk < C::BN / 16; ++kk)
          ptx::umma_ts(leader, od, pa + kk * 8, vdesc + (uint64_t)(kk * 128), C::IDESC_O, 1u);
        return true;
      };
      auto issue_s = [&](int t, uint32_t kb, int qt) {
        const uint32_t sd = tmem + t * 128;
        const uint64_t qdesc = ptx::sw128_desc(q_base + qt * C::Q_BYTES, 16, 1024);
        const uint64_t kdesc = ptx::sw128_desc(kb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * C::BLK + (kk & 3) * 32) >> 4);
          ptx::umma_ss(leader, sd, qdesc + off, kdesc + off, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        ptx::umma_commit(leader, &sh.s_full[t]);
      };
      for (uint32_t ring = 0; ok; ++ring) {
        const int slot = ring & 1;
        if (!wait(&sh.unit_full[slot], (ring >> 1) & 1)) { ok = false; break; }
        const int32_t ntiles = sh.unit[slot][U_NTILES];
        const bool two = !ALL_HALF && sh.unit[slot][U_HALF] == 0;   // second query tile active
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
        if (ntiles < 0) break;
        if (!wait(&sh.q_full, (ring & 1))) { ok = false; break; }
        // K of tile j released to the MMA: by the RoPE warps with ROPE (their barrier ring counts K tiles only:
        // a slot hosts K and V items alike, so the slot's own phase count does not apply), else by the TMA
        auto k_ready = [&](uint32_t ki) -> bool {
          return ROPE ? wait(&sh.k_rot[(ki >> 1) % NSLOT], ((ki >> 1) / NSLOT) & 1)
                      : wait(&sh.kv_full[ki % NSLOT], (ki / NSLOT) & 1);
        };
        if (SHARED_HALF && !two) {
          // half unit: tile j uses S buffer, P and O accumulator t = j & 1 over query tile 0; S_t(j) may be
          // issued once PV_t(j - 2) has been
          uint32_t v_of[2] = {0, 0};
          for (int32_t j = 0; j < ntiles && ok; ++j) {
            const int t = j & 1;
            const uint32_t ki = kv_item, vi = kv_item + 1;
            kv_item += 2;
            if (j >= 2) {
              if (!issue_pv(t, v_of[t], j < 4, true)) { ok = false; break; }
              ptx::umma_commit(leader, &sh.kv_empty[v_of[t] % NSLOT]);
            }
            if (!k_ready(ki)) { ok = false; break; }
            ptx::tc_fence_after();
            issue_s(t, kv_base + (ki % NSLOT) * C::TILE_BYTES, 0);
            ptx::umma_commit(leader, &sh.kv_empty[ki % NSLOT]);
            if (j == ntiles - 1) ptx::umma_commit(leader, &sh.q_empty);
            v_of[t] = vi;
          }
          if (!ok) break;
          // the last PV into each accumulator publishes it
          for (int32_t j = ntiles >= 2 ? ntiles - 2 : 0; j < ntiles; ++j) {
            const int t = j & 1;
            if (!issue_pv(t, v_of[t], j < 2, true)) { ok = false; break; }
            ptx::umma_commit(leader, &sh.o_full[t]);
            ptx::umma_commit(leader, &sh.kv_empty[v_of[t] % NSLOT]);
          }
          if (!ok) break;
          ++act[0];
          if (ntiles >= 2) ++act[1];
          continue;
        }
        uint32_t prev_vi = 0;
        for (int32_t j = 0; j < ntiles && ok; ++j) {
          const uint32_t ki = kv_item, vi = kv_item + 1;
          kv_item += 2;
          if (j > 0 && !issue_pv(0, prev_vi, j == 1, true)) { ok = false; break; }
          const int s = ki % NSLOT;
          if (!k_ready(ki)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t kb = kv_base + s * C::TILE_BYTES;
          issue_s(0, kb, 0);
          if (j > 0) {
            if (two && !issue_pv(1, prev_vi, j == 1, false)) { ok = false; break; }
            ptx::umma_commit(leader, &sh.kv_empty[prev_vi % NSLOT]);
          }
          if (two) issue_s(1, kb, 1);
          ptx::umma_commit(leader, &sh.kv_empty[s]);
          if (j == ntiles - 1) ptx::umma_commit(leader, &sh.q_empty);
          prev_vi = vi;
        }
        if (!ok) break;
        // the unit's last PV of each tile publishes its O
        if (!issue_pv(0, prev_vi, ntiles == 1, true)) break;
        ptx::umma_commit(leader, &sh.o_full[0]);
        if (two) {
          if (!issue_pv(1, prev_vi, ntiles == 1, false)) break;
          ptx::umma_commit(leader, &sh.o_full[1]);
        }
        ptx::umma_commit(leader, &sh.kv_empty[prev_vi % NSLOT]);
        ++act[0];
        if (two) ++act[1];
      }
      // Drain: every MMA this CTA issued has completed before tensor memory is released (a bounded wait
      // that ignores the abort flag).
      __syncwarp();
      ptx::umma_commit(leader, &sh.mma_drain);
      ptx::mbar_wait(&sh.mma_drain, 0, nullptr, status, kStatusTimeout);
      __syncwarp();
    } else if (APPEND && warp >= 10) {
      // ------------------------------------------------------------------------------ append
      // Warps 10-11 write the new keys and values of the unit's own query positions into their pool pages
      // (the positions of a (sequence, KV head) are split among its units, so every new row is written
      // once; of a split unit only the chunk that starts it writes). No CTA reads a new row from the pool:
      // new-page tiles take them from the new K/V, and the pool tile of the page holding q0 masks them.
      constexpr int VPR = D / 8;                 // 16-byte vectors per row
      const int tid = (warp - 10) * 32 + lane;   // 0 .. 63
      auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kStatusTimeout));
      };
      for (uint32_t ring = 0;; ++ring) {
        const int slot = ring & 1;
        if (!wwait(&sh.unit_full[slot], (ring >> 1) & 1)) break;
        const int32_t* u = sh.unit[slot];
        if (u[U_NTILES] < 0) {
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
          break;
        }
        if (u[U_T0] == 0 && u[U_NNEW] > 0) {
          const int32_t pos0 = u[U_POS0], nv = u[U_NPOS], qrow = u[U_QROW], kvh = u[U_KVH];
          const int32_t nsink = u[U_NSINK], w0 = u[U_W0], total = u[U_TOTAL];
          const bool is_global = u[U_GLOBAL] != 0;
          const int64_t toff = u[U_TOFF];
          for (int x = tid; x < 2 * nv * VPR; x += 64) {
            const int which = x / (nv * VPR), rest = x % (nv * VPR);
            const int32_t i = rest / VPR, vc = rest % VPR;
            const int32_t pos = pos0 + i, lp = pos / P;
            const int32_t idx = is_global ? lp : (lp < nsink ? lp : nsink + (lp - w0));
            if (idx < 0 || idx >= total || toff + idx < 0 || toff + idx >= p.page_table_len || qrow + i < 0 ||
                qrow + i >= p.total_q || kvh < 0 || kvh >= p.num_kv_heads) {
              if (status) atomicOr(status, kStatusUnit);
              continue;
            }
            const int32_t pid = p.page_table[toff + idx];
            if (pid < 0 || pid >= p.num_pages) {
              if (status) atomicOr(status, kStatusPageId);
              continue;
            }
            const int64_t src = ((int64_t)(qrow + i) * p.num_kv_heads + kvh) * D + vc * 8;
            const int64_t dst = ((int64_t)pid * P + (pos % P)) * D + vc * 8;
            *reinterpret_cast<uint4*>((which ? p.v_pool : p.k_pool) + dst) =
                *reinterpret_cast<const uint4*>((which ? p.v_new : p.k_new) + src);
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
      }
    } else if (ROPE && warp >= 12) {
      // ------------------------------------------------------------------- gather-time RoPE
      // Warps 12-15 (one per SMSP) walk the schedule like the MMA warp. Per unit they cache the sequence's
      // fragment starts in shared memory (at most kRopeSmemFragments; more are searched in global memory).
      // Each K tile, once landed, has the rows whose token falls in a fragment rotated in place (a thread
      // takes one 16-byte chunk pair in D/16 rows), is fenced for the tensor core and released through
      // k_rot.
      constexpr int CH = D / 16;                 // chunk pairs (d, d + D/2) per row
      const int tid = (warp - 12) * 32 + lane;   // 0 .. 127
      const int c = tid % CH;                    // this thread's chunk pair
      uint32_t kv_item = 0;
      auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kStatusTimeout));
      };
      auto rope_bar = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };   // the four RoPE warps
      for (uint32_t ring = 0;; ++ring) {
        const int slot = ring & 1;
        if (!wwait(&sh.unit_full[slot], (ring >> 1) & 1)) break;
        const int32_t* u = sh.unit[slot];
        const int32_t ntiles = u[U_NTILES];
        if (ntiles < 0) {
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
          break;
        }
        const int32_t t0 = u[U_T0], an = u[U_AN], b0 = u[U_B0], nsink = u[U_NSINK], w0 = u[U_W0];
        const int32_t npages = u[U_AN] + u[U_BN];
        // a sequence index outside the call (a record from another plan) rotates nothing and is reported
        const bool seq_ok = u[U_SEQ] >= 0 && u[U_SEQ] < p.num_seqs;
        if (!seq_ok && status && tid == 0) atomicOr(status, kStatusUnit);
        const int32_t flo = seq_ok ? p.frags.offs[u[U_SEQ]] : 0, fhi = seq_ok ? p.frags.offs[u[U_SEQ] + 1] : 0;
        const int32_t nfr = fhi - flo;
        const bool in_smem = nfr <= kRopeSmemFragments;
        rope_bar();                                // the previous unit's searches are done
        if (in_smem)
          for (int i = tid; i < nfr; i += 128) sh.frag_start[i] = p.frags.start[flo + i];
        rope_bar();
        const int32_t* fst = in_smem ? sh.frag_start : p.frags.start + flo;
        bool ok = true;
        for (int32_t j = 0; j < ntiles; ++j) {
          const uint32_t ki = kv_item;
          kv_item += 2;
          const int s = ki % NSLOT;
          if (!wwait(&sh.kv_full[s], (ki / NSLOT) & 1)) { ok = false; break; }
          if (nfr > 0) {
            uint8_t* tile = sKV + s * C::TILE_BYTES;
            auto token_of = [&](int32_t pos, int r) {
              const int32_t idx = pos < an ? pos : b0 + (pos - an);
              const int32_t lp = idx < nsink ? idx : w0 + (idx - nsink);
              return lp * P + (r % P);
            };
            // The tile's tokens ascend with the row (pages in logical order), so if its first and last
            // loaded rows lie in one fragment every row does: one table chunk per thread for the tile.
            const int32_t pos0 = (t0 + j) * C::PPT;
            const int32_t nld = min(C::PPT, npages - pos0);        // pages of this tile that were loaded
            const int32_t f_first = rope_fragment_of(fst, 0, nfr, token_of(pos0, 0));
            const int32_t f_last = rope_fragment_of(fst, 0, nfr, token_of(pos0 + nld - 1, nld * P - 1));
            if (f_first == f_last) {
              if (f_first >= 0) {
                const float4* t4 = reinterpret_cast<const float4*>(p.frags.cs + (int64_t)(flo + f_first) * D + 16 * c);
                const float4 t[4] = {t4[0], t4[1], t4[2], t4[3]};
#pragma unroll 1
                for (int k = 0; k < CH; ++k) {
                  const int r = tid / CH + (128 / CH) * k;
                  if (r < nld * P) rope_rotate_smem_chunk_regs<D>(tile, r, c, t);
                }
              }
            } else {
#pragma unroll 1
              for (int k = 0; k < CH; ++k) {
                const int r = tid / CH + (128 / CH) * k;
                if (r >= nld * P) continue;                // page not loaded (short last tile)
                const int32_t f = rope_fragment_of(fst, 0, nfr, token_of(pos0 + r / P, r));
                // scalar IEEE products and sums, as the build rotates (packed f32x2 forms were measured to
                // differ from them by one bf16 ulp in a few keys per 10^5)
                if (f >= 0) rope_rotate_smem_chunk<D>(tile, r, c, p.frags.cs + (int64_t)(flo + f) * D);
              }
            }
            ptx::fence_proxy_async_smem();            // the rotated rows are read by the tensor core
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.k_rot[(ki >> 1) % NSLOT]);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
    // ------------------------------------------------------------------ softmax warpgroups
    const int tile = warp >> 2;       // query tile of this warpgroup
    const int quarter = warp & 3;     // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t sbuf = tmem + tile * 128 + lane_off;
    const uint32_t obuf = tmem + 256 + tile * D + lane_off;
    const float sl2 = p.scale_log2;
    const uint64_t sl2_2 = f2_pack(sl2, sl2);
    uint32_t scount = 0;
    // completed uses of O0 and O1 (phases of o_full[0], o_full[1]) and of the half-unit hand-off, counted
    // by both warpgroups over every unit
    uint32_t o0cnt = 0, o1cnt = 0, mlcnt = 0;
    // The tcgen05.ld/st below are warp-collective, so every wait's outcome is made warp-uniform.
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort, status, kStatusTimeout));
    };
    for (uint32_t ring = 0;; ++ring) {
      const int slot = ring & 1;
      if (!wwait(&sh.unit_full[slot], (ring >> 1) & 1)) break;
      // The descriptor stays in shared memory while this unit runs: the slot is released only after
      // the epilogue, and the producer refills a slot only once every consumer has released it.
      const int32_t* u = sh.unit[slot];
      const int32_t ntiles = u[U_NTILES];
      const bool is_half = ALL_HALF || u[U_HALF] != 0;
      const bool shared_half = SHARED_HALF && is_half;           // both warpgroups on query tile 0
      const bool two_o = shared_half && ntiles >= 2;             // ... and O1 holds warpgroup 1's share
      if (ntiles < 0 || (tile == 1 && is_half && !SHARED_HALF)) {   // end of schedule, or no rows for us
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
        if (ntiles < 0) break;
        continue;
      }
      const int32_t t0 = u[U_T0];
      const int32_t pslot = (shared_half ? 0 : tile) * npos + (row >> p.log2_group);
      const bool valid_row = pslot < u[U_NPOS];
      const int32_t i_pos = u[U_POS0] + (valid_row ? pslot : u[U_NPOS] - 1);
      const int32_t head = u[U_KVH] * G + (row & (G - 1));
      const bool is_global = u[U_GLOBAL] != 0;
      const int32_t S = u[U_SINK], W = u[U_WIN];
      const int32_t npages = u[U_AN] + u[U_BN];
      const int32_t an = u[U_AN], b0 = u[U_B0], nsink = u[U_NSINK], w0 = u[U_W0];
      const int32_t noldt = u[U_NOLDT], new0 = u[U_NEW0], nnew = u[U_NNEW], splitq = u[U_SPLITQ];
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;

      for (int32_t j = shared_half ? tile : 0; j < ntiles; j += shared_half ? 2 : 1) {
        // Logical page of every slot of this KV tile, worked out before S is ready; a row needs per-column
        // bounds only if some key of the tile is invisible to it (causal edge, window edge, sink tail, a
        // short last tile, or -- appending -- the page holding q0, split between pool and new K/V).
        const int32_t tt = t0 + j;
        const bool fresh = APPEND && tt >= noldt;
        int32_t lp[C::PPT];
        bool need_mask = false;
#pragma unroll
        for (int c = 0; c < C::PPT; ++c) {
          lp[c] = -1;
          if (!fresh) {
            const int32_t x = tt * C::PPT + c;
            if (x < npages) {
              const int32_t idx = x < an ? x : b0 + (x - an);
              lp[c] = idx < nsink ? idx : w0 + (idx - nsink);
            }
          } else {
            const int32_t xn = (tt - noldt) * C::PPT + c;
            if (xn < nnew) lp[c] = new0 + xn;
          }
          if (lp[c] >= 0) {
            const int32_t j0 = lp[c] * P, j1 = j0 + P - 1;
            const bool all_vis = (j1 <= i_pos) && (is_global || j1 < S || j0 > i_pos - W) &&
                                 (!APPEND || (fresh ? j0 >= splitq : j1 < splitq));
            need_mask |= !all_vis;
          } else {
            need_mask = true;
          }
        }
        // The row's visible columns of the tile as four 32-bit words, also worked out before S is ready: per
        // page at most two column ranges (the sink part and the causal window part; one for a global head), each
        // clipped to the page and, appending, to the pool or new-K/V side of q0.
        uint32_t mw[4] = {0u, 0u, 0u, 0u};
        if (need_mask) {
          const int32_t wlo = W > i_pos ? 0 : i_pos - W + 1;   // first key of the window (key > i_pos - W)
#pragma unroll
          for (int c = 0; c < C::PPT; ++c) {
            if (lp[c] < 0) continue;
            const int32_t j0 = lp[c] * P;
            int32_t lo = 0, hi = i_pos - j0 + 1;                // causal: key <= i_pos
            if (APPEND) {
              if (fresh) lo = max(lo, splitq - j0);
              else hi = min(hi, splitq - j0);
            }
            int32_t a1 = lo, b1 = hi, a2 = 0, b2 = 0;
            if (!is_global) {
              b1 = min(hi, S - j0);                             // sink: key < S
              a2 = max(lo, wlo - j0);
              b2 = hi;
            }
            a1 = max(a1, 0) + c * P;
            b1 = min(b1, P) + c * P;
            a2 = max(a2, 0) + c * P;
            b2 = min(b2, P) + c * P;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if ((k + 1) * 32 <= c * P || k * 32 >= (c + 1) * P) continue;   // compile-time: the page's words
              mw[k] |= range_bits(a1 - 32 * k, b1 - 32 * k) | range_bits(a2 - 32 * k, b2 - 32 * k);
            }
          }
        }
        if (!wwait(&sh.s_full[tile], scount & 1)) { ok = false; break; }
        ++scount;
        ptx::tc_fence_after();
        // S row in two halves: the second half's TMEM load overlaps the first half's masking and max.
        float s[128];
        ptx::tmem_ld32(sbuf, reinterpret_cast<uint32_t*>(s));
        ptx::tmem_ld32(sbuf + 32, reinterpret_cast<uint32_t*>(s) + 32);
        ptx::tmem_ld_wait();
        ptx::tmem_ld32(sbuf + 64, reinterpret_cast<uint32_t*>(s) + 64);
        ptx::tmem_ld32(sbuf + 96, reinterpret_cast<uint32_t*>(s) + 96);

        // Row max as eight independent 3-input max chains per half, so no long dependency chain.
        float mh[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1) ptx::tmem_ld_wait();
          if (need_mask) {
#pragma unroll
            for (int k = 0; k < 64; ++k) {
              const int col = h * 64 + k;                // compile-time word and bit
              if (!((mw[col >> 5] >> (col & 31)) & 1u)) s[col] = -INFINITY;
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int b = h * 64 + k * 16;
            float a = fmax3(s[b], s[b + 1], s[b + 2]);
            a = fmax3(a, s[b + 3], s[b + 4]);
            a = fmax3(a, s[b + 5], s[b + 6]);
            a = fmax3(a, s[b + 7], s[b + 8]);
            a = fmax3(a, s[b + 9], s[b + 10]);
            a = fmax3(a, s[b + 11], s[b + 12]);
            a = fmax3(a, s[b + 13], s[b + 14]);
            mh[h * 4 + k] = fmaxf(a, s[b + 15]);
          }
        }
        const float mx = fmaxf(fmax3(mh[0], mh[1], mh[2]), fmax3(fmax3(mh[3], mh[4], mh[5]), mh[6], mh[7]));
        const float m_tile = mx * sl2;
        const float m_new = fmaxf(m_run, m_tile);
        bool resc = false;
        if (j == 0 || (SHARED_HALF && m_run == -INFINITY)) {
          // No visible key of this row so far: O_t holds nothing of it (zeros, or the previous unit's values
          // that the first P V overwrites), so nothing is rescaled. On a shared half unit this must not touch
          // O1 at all: warpgroup 1 starts at tile 1 while warpgroup 0 may still be reading the previous
          // unit's O1 for its merge.
          m_run = m_new;
        } else {
          resc = m_new > m_run + 8.0f;
        }
        const float alpha = resc ? ptx::ex2(m_run - m_new) : 1.0f;
        if (resc) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float mu = (m_run == -INFINITY) ? 0.f : m_run;
        const uint64_t nmu2 = f2_pack(-mu, -mu);
        uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {          // two halves of 64 keys -> 32 packed P columns each
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int e = h * 64 + 2 * c;
            const uint64_t x2 = f2_fma(f2_pack(s[e], s[e + 1]), sl2_2, nmu2);
            uint64_t p2;
            if (kExpCubicEvery > 0 && c % kExpCubicEvery == kExpCubicEvery - 1) {
              p2 = exp2_cubic_pair(x2);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p2 = f2_pack(ptx::ex2(x0), ptx::ex2(x1));
            }
            sum2[c & 3] = f2_add(sum2[c & 3], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            pk[c] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st32(sbuf + h * 32, pk);
          if (h == 0 && __any_sync(0xffffffffu, resc)) {
            // Rescale O_t in place before any of P_t(j) is published (the first half of S is dead by now,
            // which leaves registers for it). O_t holds every PV issued so far -- the commit that published
            // S_t(j) covered PV_t(j-1) -- and PV_t(j) waits for this warp's arrivals.
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              ptx::tmem_ld32(obuf + c * 32, r);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), a2), lo, hi);
                r[2 * k] = __float_as_uint(lo);
                r[2 * k + 1] = __float_as_uint(hi);
              }
              ptx::tmem_st32(obuf + c * 32, r);
            }
          }
          // publish this half of P_t(j): the first lets the MMA warp start on keys 0-63
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(h == 0 ? &sh.p_half[tile] : &sh.p_full[tile]);
        }
        float sa, sb;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sa, sb);
        l_run += sa + sb;
      }
      if (!ok) break;

      // ------------------------------------------------------------------------------ epilogue
      if (shared_half && tile == 1) {
        // hand the running max and sum of warpgroup 1's KV tiles to warpgroup 0, which merges
        if (two_o) {
          // the previous hand-off has been read
          if (!wwait(&sh.ml_empty, (mlcnt & 1) ^ 1)) break;
          sh.ml[2 * row] = m_run;
          sh.ml[2 * row + 1] = l_run;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh.ml_full);
          ++o1cnt;
          ++mlcnt;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.unit_empty[slot]);
        continue;
      }
      if (!wwait(&sh.o_full[tile], (tile == 0 ? o0cnt : o1cnt) & 1)) break;
      // weights of the two accumulators: (1, 0) unless this is a shared half unit with two shares
      float a0 = 1.f, a1 = 0.f;
      if (two_o) {
        if (!wwait(&sh.ml_full, mlcnt & 1) || !wwait(&sh.o_full[1], o1cnt & 1)) break;
        const float m1 = sh.ml[2 * row], l1 = sh.ml[2 * row + 1];
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.ml_empty);
        const float M = fmaxf(m_run, m1);
        a0 = (m_run == -INFINITY) ? 0.f : ptx::ex2(m_run - M);
        a1 = (m1 == -INFINITY) ? 0.f : ptx::ex2(m1 - M);
        l_run = a0 * l_run + a1 * l1;
        m_run = M;
      }
      const uint32_t obuf1 = tmem + 256 + D + lane_off;   // O1, merged into O0's rows
      ptx::tc_fence_after();
      // O columns [64 h, 64 h + 64) of this warpgroup's rows (two loads, one wait), merged with O1 for a shared
      // half unit
      auto load_o = [&](int h, uint32_t (&r)[64]) {
        ptx::tmem_ld32(obuf + h * 64, r);
        ptx::tmem_ld32(obuf + h * 64 + 32, r + 32);
        if (two_o) {
          uint32_t r1[64];
          ptx::tmem_ld32(obuf1 + h * 64, r1);
          ptx::tmem_ld32(obuf1 + h * 64 + 32, r1 + 32);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 64; ++k)
            r[k] = __float_as_uint(__fmaf_rn(a1, __uint_as_float(r1[k]), a0 * __uint_as_float(r[k])));
        } else {
          ptx::tmem_ld_wait();
        }
      };
      auto release = [&] {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&sh.o_free[tile]);
          if (two_o) ptx::mbar_arrive(&sh.o_free[1]);   // warpgroup 0 read O1 too
          ptx::mbar_arrive(&sh.unit_empty[slot]);
        }
        ++o0cnt;                                   // every unit publishes O0
        if (!is_half || two_o) ++o1cnt;            // full units and shared half units with two shares, O1
        if (two_o) ++mlcnt;
      };
      const int32_t part = u[U_PART];
      if (part >= 0) {
        // one chunk of a split unit: O / l in fp32 and the chunk's LSE, for the combine pass; a row that
        // saw no visible key in this chunk writes O = 0 and LSE = -inf. A slot the workspace does not have
        // (a record from another plan) is skipped and reported.
        const bool empty = (m_run == -INFINITY) || !(l_run > 0.f);
        const float inv_l = empty ? 0.f : 1.0f / l_run;
        const bool slot_ok = part < p.num_partials;
        if (!slot_ok && status && quarter == 0 && lane == 0) atomicOr(status, kStatusUnit);
        const int32_t prow = tile * 128 + row;
        float4* dst = reinterpret_cast<float4*>(p.part_o);
#pragma unroll 1
        for (int h = 0; h < D / 64; ++h) {
          uint32_t r[64];
          load_o(h, r);
          if (slot_ok) {
#pragma unroll
            for (int k = 0; k < 16; ++k)   // 4-column groups 16h .. 16h + 15, coalesced over the warp's rows
              dst[partial_o_index<D>(part, prow, h * 16 + k)] =
                  make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                              __uint_as_float(r[4 * k + 2]) * inv_l, __uint_as_float(r[4 * k + 3]) * inv_l);
          }
        }
        if (slot_ok) p.part_lse[(int64_t)part * 256 + prow] = empty ? -INFINITY : (m_run + __log2f(l_run)) * 0.69314718055994531f;
        release();
        continue;
      }
      const float inv_l = 1.0f / l_run;
      const int64_t qrow = (int64_t)u[U_QROW] + pslot;
      // a row or head outside the call's outputs (a record from another plan) is skipped and reported
      const bool in_range = qrow >= 0 && qrow < p.total_q && head >= 0 && head < p.num_q_heads;
      if (valid_row && !in_range && status) atomicOr(status, kStatusUnit);
      const bool store_row = valid_row && in_range;
      __nv_bfloat16* orow = p.o + (qrow * p.num_q_heads + head) * D;
      // 32-byte stores when O is 32-byte aligned (every row then is: rows are D x 2 bytes apart)
      const bool v8 = (reinterpret_cast<uintptr_t>(p.o) & 31) == 0;
#pragma unroll 1
      for (int h = 0; h < D / 64; ++h) {
        uint32_t r[64];
        load_o(h, r);
        uint32_t w[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          w[k] = ptx::pack_bf16x2(__uint_as_float(r[2 * k]) * inv_l, __uint_as_float(r[2 * k + 1]) * inv_l);
        if (store_row) {
          if (v8) {
#pragma unroll
            for (int k = 0; k < 4; ++k) ptx::st_global_v8(orow + h * 64 + k * 16, w + 8 * k);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + h * 64);
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
      if (store_row) p.lse[(int64_t)head * p.total_q + qrow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      release();
    }
  }

  // ------------------------------------------------------------------------------------ teardown
  // Every warp arrives at the block barrier converged (the roles leave their loops after lane-0-only
  // arrivals), so each warp is counted once and tensor memory is released only after every role is done.
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace segpaged
