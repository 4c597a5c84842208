// combine_kernel.cuh -- merges the chunks of split prefill units.
//
// A long unit whose KV tiles are spread over several CTAs leaves one partial result per chunk: O_c = the
// chunk's softmax-weighted V sum normalised by its own row sum, and LSE_c, the natural-log sum of the
// chunk's exponentials (-inf when the row saw no visible key in it). Exact attention over the union is
//   LSE = log sum_c exp(LSE_c),   O = sum_c exp(LSE_c - LSE) O_c.
// One pass per row merges the chunks online (running max, rescaled sum and accumulator), in chunk order, so
// the result depends only on the plan, never on which CTA ran which chunk. Partials are stored column-group
// major (partial_o_group): a warp's 32 consecutive rows of one 4-column group are 512 contiguous bytes, so
// both the prefill's stores and the loads here are coalesced. A block takes 32 rows of a record; for a record
// of at most 16 chunks its eight warps take eight column ranges of every chunk, for a wider one the block
// takes one column range (grid z) and its eight warps take every eighth chunk, merged in warp order.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"

namespace segpaged {

constexpr int kCombineMaxSplit = 256;  // chunks per unit (the planner never makes more)
constexpr int kCombineWideSplit = 16;  // records with more chunks split their chunks over a block's warps
constexpr int kCombineRows = 256;      // rows of a combine record (two query tiles)
constexpr int kCombineBlockRows = 32;  // rows of one combine block (a lane each)
constexpr int32_t kCombineStatusUnit = 8;   // SEGPAGED_STATUS_UNIT: the grid had too few row blocks

// Row blocks of 32 rows the combine launch needs for one record: up to its last valid row (a query tile
// holds 128/G positions x G heads, the second tile from row 128).
SP_HD int64_t combine_blocks_of(int32_t npos, int32_t nsplit, int32_t G) {
  (void)nsplit;
  const int32_t npos_tile = 128 / G;
  const int32_t rows = npos <= npos_tile ? npos * G : 128 + (npos - npos_tile) * G;
  return ceil_div(rows, kCombineBlockRows);
}

// The float4 of 4-column group `group` of row `row` of partial slot `slot` (slots of 256 rows x D columns).
template <int D>
__device__ __forceinline__ size_t partial_o_index(int64_t slot, int32_t row, int32_t group) {
  return (size_t)((slot * (D / 4) + group) * 256 + row);
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct CombineParams {
  const int32_t* records;  // combine records [num_groups][U_NFIELDS]
  int32_t num_groups;
  const float* part_o;     // [slots][D/4][256] float4 groups (partial_o_index)
  const float* part_lse;   // [slots][256]
  __nv_bfloat16* o;        // [total_q, Hq, D]
  float* lse;              // [Hq, total_q]
  int32_t total_q, num_q_heads, log2_group;
  int32_t num_partials;    // partial slots in part_o / part_lse
  int32_t row_blocks;      // gridDim.y: the most row blocks a record needs
  int32_t* status;         // nullable
};

// Online merge of chunks c = c0, c0 + stride, ... of one row into (m, wsum, acc) for GW column groups from
// group g0: the loads of four chunks are issued together, the running max rescales what was accumulated so
// far when it grows.
template <int D, int GW>
__device__ __forceinline__ void merge_chunks(const float4* part_o, const float* part_lse, int32_t part0,
                                             int32_t nsplit, int c0, int stride, int r, int g0, float& m,
                                             float& wsum, float (&acc)[4 * GW]) {
  constexpr int NB = 4;
  for (int c = c0; c < nsplit; c += NB * stride) {
    float lc[NB];
    float4 v[NB][GW];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int cc = c + u * stride;
      lc[u] = -INFINITY;
      if (cc < nsplit) {
        const int64_t slot = part0 + cc;
        lc[u] = part_lse[slot * 256 + r];
#pragma unroll
        for (int g = 0; g < GW; ++g) v[u][g] = part_o[partial_o_index<D>(slot, r, g0 + g)];
      }
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      if (lc[u] == -INFINITY) continue;  // no visible key of this row in the chunk (or past the end)
      if (lc[u] > m) {
        const float f = (m == -INFINITY) ? 0.f : expf(m - lc[u]);
        wsum *= f;
#pragma unroll
        for (int k = 0; k < 4 * GW; ++k) acc[k] *= f;
        m = lc[u];
      }
      const float w = expf(lc[u] - m);
      wsum += w;
#pragma unroll
      for (int g = 0; g < GW; ++g) {
        acc[4 * g] += w * v[u][g].x;
        acc[4 * g + 1] += w * v[u][g].y;
        acc[4 * g + 2] += w * v[u][g].z;
        acc[4 * g + 3] += w * v[u][g].w;
      }
    }
  }
}

// grid: (combine records, row blocks of 32 rows: as many as the widest record needs, D / (4 GW) column ranges).
// A record of at most 16 chunks is merged by the z = 0 blocks, warp w taking column groups [w GW, w GW + GW)
// of every chunk; a wider record by all z, block z taking column groups [z GW, z GW + GW) and warp w the
// chunks c = w (mod 8), the eight partial triples merged in order 0..7 through shared memory.
template <int D>
__global__ void __launch_bounds__(256) segpaged_combine_kernel(const CombineParams p) {
  constexpr int NW = 8;           // warps per block
  constexpr int GW = D / 32;      // 4-column groups per warp (D / 4 groups over 8 warps)
  __shared__ float s_m[NW][32], s_sum[NW][32];
  __shared__ float s_acc[NW][4 * GW][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = 1 << p.log2_group;
  const int npos_tile = 128 >> p.log2_group;
  const float4* part_o = reinterpret_cast<const float4*>(p.part_o);
  for (int gi = blockIdx.x; gi < p.num_groups; gi += gridDim.x) {
    const int32_t* rec = p.records + (int64_t)gi * U_NFIELDS;
    const int32_t part0 = rec[U_PART], nsplit = rec[U_NSPLIT], npos = rec[U_NPOS];
    const int32_t qrow0 = rec[U_QROW], kvh = rec[U_KVH];
    const int rows = rec[U_HALF] ? 128 : 256;
    const bool wide = nsplit > kCombineWideSplit;
    // the last row block checks that the grid reaches every valid row of the record
    if (blockIdx.y == gridDim.y - 1 && blockIdx.z == 0 && threadIdx.x == 0 && p.status &&
        combine_blocks_of(npos, nsplit, G) > (int64_t)gridDim.y)
      atomicOr(p.status, kCombineStatusUnit);
    // a record whose slots, rows or heads fall outside the call's arrays (not from this call's plan) is
    // skipped and reported
    if (part0 < 0 || nsplit < 0 || (int64_t)part0 + nsplit > p.num_partials || qrow0 < 0 ||
        (int64_t)qrow0 + npos > p.total_q || (int64_t)(kvh + 1) * G > p.num_q_heads) {
      if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && p.status) atomicOr(p.status, kCombineStatusUnit);
      continue;
    }
    if ((!wide && blockIdx.z != 0) || (int)blockIdx.y * kCombineBlockRows >= rows) continue;   // uniform
    const int r = (int)blockIdx.y * kCombineBlockRows + lane;
    const int tile = r >> 7, rr = r & 127;
    const int32_t pslot = tile * npos_tile + (rr >> p.log2_group);
    const bool active = r < rows && pslot < npos;
    const int g0 = (wide ? (int)blockIdx.z : warp) * GW;
    float m = -INFINITY, wsum = 0.f, acc[4 * GW];
#pragma unroll
    for (int k = 0; k < 4 * GW; ++k) acc[k] = 0.f;
    if (active) merge_chunks<D, GW>(part_o, p.part_lse, part0, nsplit, wide ? warp : 0, wide ? NW : 1, r, g0, m, wsum, acc);
    if (wide) {
      s_m[warp][lane] = m;
      s_sum[warp][lane] = wsum;
#pragma unroll
      for (int k = 0; k < 4 * GW; ++k) s_acc[warp][k][lane] = acc[k];
      __syncthreads();
      if (warp == 0) {
        float M = s_m[0][lane];
#pragma unroll
        for (int q = 1; q < NW; ++q) M = fmaxf(M, s_m[q][lane]);
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < 4 * GW; ++k) acc[k] = 0.f;
#pragma unroll
        for (int q = 0; q < NW; ++q) {
          const float f = (s_m[q][lane] == -INFINITY) ? 0.f : expf(s_m[q][lane] - M);
          tot += f * s_sum[q][lane];
#pragma unroll
          for (int k = 0; k < 4 * GW; ++k) acc[k] += f * s_acc[q][k][lane];
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
      __nv_bfloat16* dst = p.o + (qrow * p.num_q_heads + head) * D + g0 * 4;
#pragma unroll
      for (int k = 0; k < 4 * GW; k += 8) {
        uint4 w;
        w.x = pack2_bf16(acc[k] * inv, acc[k + 1] * inv);
        w.y = pack2_bf16(acc[k + 2] * inv, acc[k + 3] * inv);
        w.z = pack2_bf16(acc[k + 4] * inv, acc[k + 5] * inv);
        w.w = pack2_bf16(acc[k + 6] * inv, acc[k + 7] * inv);
        *reinterpret_cast<uint4*>(dst + k) = w;
      }
      if (g0 == 0) p.lse[(int64_t)head * p.total_q + qrow] = m + logf(wsum);
    }
  }
}

}  // namespace segpaged
