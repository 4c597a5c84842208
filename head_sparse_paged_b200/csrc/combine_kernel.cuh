// combine_kernel.cuh -- merges the chunks of split prefill units.
//
// A long unit whose KV tiles are spread over several CTAs leaves one partial result per chunk: O_c = the
// chunk's softmax-weighted V sum normalised by its own row sum, and LSE_c, the natural-log sum of the
// chunk's exponentials (-inf when the row saw no visible key in it). Exact attention over the union is
//   LSE = log sum_c exp(LSE_c),   O = sum_c exp(LSE_c - LSE) O_c.
// One pass per row merges the chunks online (running max, rescaled sum and accumulator), eight chunks'
// loads in flight at a time; rows of records with few chunks get a warp each, rows of records with many
// chunks a whole block whose eight per-warp results (four loads in flight each) are merged in a fixed order. The order of the merge
// depends only on the plan, never on which CTA ran which chunk. Each lane owns D/32 columns (coalesced).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"

namespace segpaged {

constexpr int kCombineMaxSplit = 256;  // chunks per unit (the planner never makes more)
constexpr int kCombineWideSplit = 16;  // records with more chunks get a block per row, the others a warp
constexpr int kCombineRows = 256;      // rows of a combine record (two query tiles)
constexpr int32_t kCombineStatusUnit = 8;   // SEGPAGED_STATUS_UNIT: the grid had too few row blocks

// Thread blocks the combine launch needs for one record: up to its last valid row (a query tile holds
// 128/G positions x G heads, the second tile from row 128), one block per row for a wide record, one per
// 8 rows otherwise.
SP_HD int64_t combine_blocks_of(int32_t npos, int32_t nsplit, int32_t G) {
  const int32_t npos_tile = 128 / G;
  const int32_t rows = npos <= npos_tile ? npos * G : 128 + (npos - npos_tile) * G;
  return nsplit > kCombineWideSplit ? rows : ceil_div(rows, 8);
}

struct CombineParams {
  const int32_t* records;  // combine records [num_groups][U_NFIELDS]
  int32_t num_groups;
  const float* part_o;     // [slots][256][D]
  const float* part_lse;   // [slots][256]
  __nv_bfloat16* o;        // [total_q, Hq, D]
  float* lse;              // [Hq, total_q]
  int32_t total_q, num_q_heads, log2_group;
  int32_t num_partials;    // partial slots in part_o / part_lse
  int32_t row_blocks;      // gridDim.y: the most row blocks a record needs
  int32_t* status;         // nullable
};

// Online merge of chunks c = c0, c0 + stride, ... into (m, wsum, acc): the loads of NB chunks are issued
// together (one round trip for a record of up to NB chunks), the running max rescales what was accumulated
// so far when it grows.
template <int V, int NB>
__device__ __forceinline__ void merge_chunks(const float* part_o, const float* part_lse, int32_t part0, int32_t nsplit,
                                             int c0, int stride, int r, int lane, int D, float& m, float& wsum,
                                             float (&acc)[V]) {
  int c = c0;
  for (; c < nsplit; c += NB * stride) {
    float lc[NB];
    float2 v[NB][V / 2];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int cc = c + u * stride;
      lc[u] = -INFINITY;
      if (cc < nsplit) {
        const int64_t slot = part0 + cc;
        lc[u] = part_lse[slot * 256 + r];
        const float* src = part_o + (slot * 256 + r) * D + lane * V;
#pragma unroll
        for (int k = 0; k < V / 2; ++k) v[u][k] = *reinterpret_cast<const float2*>(src + 2 * k);
      }
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      if (lc[u] == -INFINITY) continue;  // no visible key of this row in the chunk (or past the end)
      if (lc[u] > m) {
        const float f = (m == -INFINITY) ? 0.f : expf(m - lc[u]);
        wsum *= f;
#pragma unroll
        for (int k = 0; k < V; ++k) acc[k] *= f;
        m = lc[u];
      }
      const float w = expf(lc[u] - m);
      wsum += w;
#pragma unroll
      for (int k = 0; k < V / 2; ++k) {
        acc[2 * k] += w * v[u][k].x;
        acc[2 * k + 1] += w * v[u][k].y;
      }
    }
  }
}

// grid: (combine records, row blocks: as many as the widest record needs, at most 256). A record with at
// most 16 chunks gets one warp per row (blockIdx.y picks a block of 8 rows); a wider record gets all 8
// warps of a block on one row (blockIdx.y is the row), warp w merging chunks c = w (mod 8), and the eight
// partial triples are merged in order 0..7.
template <int D>
__global__ void __launch_bounds__(256) segpaged_combine_kernel(const CombineParams p) {
  constexpr int V = D / 32;  // columns per lane
  constexpr int NW = 8;      // warps per block
  __shared__ float s_m[NW], s_sum[NW];
  __shared__ float s_acc[NW][D];
  // Launched as a programmatic dependent of the prefill: wait until that grid has completed and its
  // partial results are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = 1 << p.log2_group;
  const int npos_tile = 128 >> p.log2_group;
  for (int gi = blockIdx.x; gi < p.num_groups; gi += gridDim.x) {
    const int32_t* rec = p.records + (int64_t)gi * U_NFIELDS;
    const int32_t part0 = rec[U_PART], nsplit = rec[U_NSPLIT], npos = rec[U_NPOS];
    const int32_t qrow0 = rec[U_QROW], kvh = rec[U_KVH];
    const int rows = rec[U_HALF] ? 128 : 256;
    const bool wide = nsplit > kCombineWideSplit;
    // the last row block checks that the grid reaches every valid row of the record
    if (blockIdx.y == gridDim.y - 1 && threadIdx.x == 0 && p.status &&
        combine_blocks_of(npos, nsplit, G) > (int64_t)gridDim.y)
      atomicOr(p.status, kCombineStatusUnit);
    // a record whose slots, rows or heads fall outside the call's arrays (not from this call's plan) is
    // skipped and reported
    if (part0 < 0 || nsplit < 0 || (int64_t)part0 + nsplit > p.num_partials || qrow0 < 0 ||
        (int64_t)qrow0 + npos > p.total_q || (int64_t)(kvh + 1) * G > p.num_q_heads) {
      if (blockIdx.y == 0 && threadIdx.x == 0 && p.status) atomicOr(p.status, kCombineStatusUnit);
      continue;
    }
    const int r = wide ? (int)blockIdx.y : (int)blockIdx.y * NW + warp;
    if ((wide ? r : (int)blockIdx.y * NW) >= rows) continue;     // uniform for the whole block
    const int tile = r >> 7, rr = r & 127;
    const int32_t pslot = tile * npos_tile + (rr >> p.log2_group);
    const bool active = r < rows && pslot < npos;
    if (wide && !active) continue;                                // uniform: one row per block
    float m = -INFINITY, wsum = 0.f, acc[V];
#pragma unroll
    for (int k = 0; k < V; ++k) acc[k] = 0.f;
    if (active) {
      if (wide) merge_chunks<V, 4>(p.part_o, p.part_lse, part0, nsplit, warp, NW, r, lane, D, m, wsum, acc);
      else merge_chunks<V, 8>(p.part_o, p.part_lse, part0, nsplit, 0, 1, r, lane, D, m, wsum, acc);
    }
    if (wide) {
      if (lane == 0) {
        s_m[warp] = m;
        s_sum[warp] = wsum;
      }
#pragma unroll
      for (int k = 0; k < V; ++k) s_acc[warp][lane * V + k] = acc[k];
      __syncthreads();
      if (warp == 0) {
        float M = s_m[0];
#pragma unroll
        for (int q = 1; q < NW; ++q) M = fmaxf(M, s_m[q]);
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < V; ++k) acc[k] = 0.f;
#pragma unroll
        for (int q = 0; q < NW; ++q) {
          const float f = (s_m[q] == -INFINITY) ? 0.f : expf(s_m[q] - M);
          tot += f * s_sum[q];
#pragma unroll
          for (int k = 0; k < V; ++k) acc[k] += f * s_acc[q][lane * V + k];
        }
        m = M;
        wsum = tot;
      }
      __syncthreads();
    }
    if (active && (!wide || warp == 0)) {
      const float inv = 1.0f / wsum;
      const int32_t head = kvh * G + (rr & (G - 1));
      const int64_t qrow = (int64_t)qrow0 + pslot;
      __nv_bfloat16* dst = p.o + (qrow * p.num_q_heads + head) * D + lane * V;
#pragma unroll
      for (int k = 0; k < V; k += 2)
        *reinterpret_cast<__nv_bfloat162*>(dst + k) = __floats2bfloat162_rn(acc[k] * inv, acc[k + 1] * inv);
      if (lane == 0) p.lse[(int64_t)head * p.total_q + qrow] = m + logf(wsum);
    }
  }
}

}  // namespace segpaged
