// topk_kernel.cuh -- per-sequence top-k tokens by attention mass (the sparse-FFN selection).
//
// One block per sequence. Masses are finite and >= 0, so their bit patterns order like the values:
// a radix select over the 32 bits (four 8-bit digits, shared-memory histograms) finds the k-th
// largest value T and how many of the values equal to T are still needed. A final pass in row order
// keeps every row above T and the first needed rows equal to T (the lower row wins a tie), writing
// them in ascending row order through block-wide prefix sums.
#pragma once
#include <stdint.h>

namespace segpaged {

constexpr int kTopkThreads = 1024;

// Exclusive prefix sum over the block of one value per thread; *total receives the block sum.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) warp_sums[lane] = w;   // inclusive warp prefix
  }
  __syncthreads();
  const int32_t before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[nw - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kTopkThreads) topk_select_kernel(const float* __restrict__ mass,
                                                                  const int32_t* __restrict__ cu_q,
                                                                  const int32_t* __restrict__ k_per_seq,
                                                                  int32_t* __restrict__ selected) {
  __shared__ int32_t hist[256];
  __shared__ int32_t warp_sums[32];
  __shared__ uint32_t s_prefix, s_need;
  __shared__ int64_t s_off;
  const int b = blockIdx.x;
  const int32_t lo = cu_q[b], n = cu_q[b + 1] - lo;
  auto clamp_k = [&](int c) {
    const int32_t nc = cu_q[c + 1] - cu_q[c];
    return min(max(k_per_seq[c], 0), max(nc, 0));
  };
  // offset of this sequence's list: the chosen counts of the sequences before it
  if (threadIdx.x < 32) {
    int64_t acc = 0;
    for (int c = threadIdx.x; c < b; c += 32) acc += clamp_k(c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (threadIdx.x == 0) s_off = acc;
  }
  __syncthreads();
  const int32_t kb = clamp_k(b);
  const int64_t off = s_off;
  if (kb == 0) return;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(mass + lo);
  if (kb == n) {
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) selected[off + i] = lo + i;
    return;
  }
  uint32_t prefix = 0, mask = 0, need = (uint32_t)kb;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t u = bits[i];
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t above = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (above + (uint32_t)hist[d] >= need) break;
        above += (uint32_t)hist[d];
      }
      s_prefix = prefix | ((uint32_t)d << shift);
      s_need = need - above;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix is now the k-th largest value T; `need` of the rows equal to T are kept, lowest first.
  int32_t eq_before = 0, out_before = 0;
  for (int32_t base = 0; base < n; base += blockDim.x) {
    const int32_t i = base + threadIdx.x;
    const uint32_t u = i < n ? bits[i] : 0u;
    const int32_t gt = (i < n && u > prefix) ? 1 : 0;
    const int32_t eq = (i < n && u == prefix) ? 1 : 0;
    int32_t eq_total, take_total;
    const int32_t eq_rank = eq_before + block_exclusive_scan(eq, warp_sums, &eq_total);
    const int32_t take = gt | (eq & (eq_rank < (int32_t)need ? 1 : 0));
    const int32_t pos = out_before + block_exclusive_scan(take, warp_sums, &take_total);
    if (take) selected[off + pos] = lo + i;
    eq_before += eq_total;
    out_before += take_total;
  }
}

}  // namespace segpaged
