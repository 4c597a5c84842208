// combine_kernel.cuh -- merges the chunks of split prefill units.
//
// A long unit whose KV tiles are spread over several CTAs leaves one partial result per chunk: O_c = the
// chunk's softmax-weighted V sum normalised by its own row sum, and LSE_c, the natural-log sum of the
// chunk's exponentials (-inf when the row saw no visible key in it). Exact attention over the union is
//   LSE = log sum_c exp(LSE_c),   O = sum_c exp(LSE_c - LSE) O_c.
// A block handles two tile rows of one combine record with four warps per row: warp part k takes the
// chunks c = k (mod 4) (loads unrolled for memory-level parallelism) and keeps its own (max, sum, O)
// triple; the four triples are then merged in a fixed order, so the result does not depend on which CTA
// ran which chunk. Each lane owns D/32 columns (coalesced). HBM-bound and small.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"

namespace segpaged {

constexpr int kCombineMaxSplit = 256;  // chunks per unit (the planner never makes more)

struct CombineParams {
  const int32_t* records;  // combine records [num_groups][U_NFIELDS]
  int32_t num_groups;
  const float* part_o;     // [slots][256][D]
  const float* part_lse;   // [slots][256]
  __nv_bfloat16* o;        // [total_q, Hq, D]
  float* lse;              // [Hq, total_q]
  int32_t total_q, num_q_heads, log2_group;
};

// grid: (combine records, 128 row pairs); block: 256 threads = 2 rows x 4 warps.
template <int D>
__global__ void __launch_bounds__(256) segpaged_combine_kernel(const CombineParams p) {
  constexpr int V = D / 32;  // columns per lane
  __shared__ float s_m[2][4], s_sum[2][4];
  __shared__ float s_acc[2][4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = warp >> 2, part = warp & 3;  // row within the block, chunk residue of this warp
  const int G = 1 << p.log2_group;
  const int npos_tile = 128 >> p.log2_group;
  for (int gi = blockIdx.x; gi < p.num_groups; gi += gridDim.x) {
    const int32_t* rec = p.records + (int64_t)gi * U_NFIELDS;
    const int32_t part0 = rec[U_PART], nsplit = rec[U_NSPLIT], npos = rec[U_NPOS];
    const int32_t qrow0 = rec[U_QROW], kvh = rec[U_KVH];
    const int rows = rec[U_HALF] ? 128 : 256;
    const int r = blockIdx.y * 2 + rl;
    const int tile = r >> 7, rr = r & 127;
    const int32_t pslot = tile * npos_tile + (rr >> p.log2_group);
    const bool active = r < rows && pslot < npos;    // uniform per row (per warp group of 4)
    float m = -INFINITY, wsum = 0.f, acc[V];
#pragma unroll
    for (int k = 0; k < V; ++k) acc[k] = 0.f;
    if (active) {
      // this warp's chunks: c = part + 4 * t, t = 0, 1, ...
      for (int c = part + 4 * lane; c < nsplit; c += 128) m = fmaxf(m, p.part_lse[(int64_t)(part0 + c) * 256 + r]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (m != -INFINITY) {
        int c = part;
        for (; c + 12 < nsplit; c += 16) {   // four chunks in flight per iteration
          float lc[4];
          float2 v[4][V / 2];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int64_t slot = part0 + c + 4 * u;
            lc[u] = p.part_lse[slot * 256 + r];
            const float* src = p.part_o + (slot * 256 + r) * D + lane * V;
#pragma unroll
            for (int k = 0; k < V / 2; ++k) v[u][k] = *reinterpret_cast<const float2*>(src + 2 * k);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float w = (lc[u] == -INFINITY) ? 0.f : expf(lc[u] - m);
            wsum += w;
#pragma unroll
            for (int k = 0; k < V / 2; ++k) {
              acc[2 * k] += w * v[u][k].x;
              acc[2 * k + 1] += w * v[u][k].y;
            }
          }
        }
        for (; c < nsplit; c += 4) {
          const float lc = p.part_lse[(int64_t)(part0 + c) * 256 + r];
          if (lc == -INFINITY) continue;  // no visible key of this row in the chunk
          const float w = expf(lc - m);
          wsum += w;
          const float* src = p.part_o + ((int64_t)(part0 + c) * 256 + r) * D + lane * V;
#pragma unroll
          for (int k = 0; k < V; k += 2) {
            const float2 vv = *reinterpret_cast<const float2*>(src + k);
            acc[k] += w * vv.x;
            acc[k + 1] += w * vv.y;
          }
        }
      }
    }
    if (lane == 0) {
      s_m[rl][part] = m;
      s_sum[rl][part] = wsum;
    }
#pragma unroll
    for (int k = 0; k < V; ++k) s_acc[rl][part][lane * V + k] = acc[k];
    __syncthreads();
    if (active && part == 0) {
      // merge the four warps' triples in order 0..3
      float M = s_m[rl][0];
#pragma unroll
      for (int q = 1; q < 4; ++q) M = fmaxf(M, s_m[rl][q]);
      float tot = 0.f, out[V];
#pragma unroll
      for (int k = 0; k < V; ++k) out[k] = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f = (s_m[rl][q] == -INFINITY) ? 0.f : expf(s_m[rl][q] - M);
        tot += f * s_sum[rl][q];
#pragma unroll
        for (int k = 0; k < V; ++k) out[k] += f * s_acc[rl][q][lane * V + k];
      }
      const float inv = 1.0f / tot;
      const int32_t head = kvh * G + (rr & (G - 1));
      const int64_t qrow = (int64_t)qrow0 + pslot;
      __nv_bfloat16* dst = p.o + (qrow * p.num_q_heads + head) * D + lane * V;
#pragma unroll
      for (int k = 0; k < V; k += 2)
        *reinterpret_cast<__nv_bfloat162*>(dst + k) = __floats2bfloat162_rn(out[k] * inv, out[k + 1] * inv);
      if (lane == 0) p.lse[(int64_t)head * p.total_q + qrow] = M + logf(tot);
    }
    __syncthreads();
  }
}

}  // namespace segpaged
