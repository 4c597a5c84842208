// build_kernel.cuh -- BUILDSTATE: scatter a layer's dense K/V into the SegPaged page pools.
//
// Each stored page of each (sequence, KV head) is one work item (a grid-stride loop over the
// flattened page tables). A block copies the page's P rows of K and V with 16-byte loads and stores,
// coalesced along D; rows past the context end are written as zero. With a RoPE table, each key is
// rotated from its original position to its actual one (shshi.cn, 技术原理 2 "位置无关缓存复用",
// item "RoPE位置对齐"): rotate-half pairs (d, d + D/2), y1 = x1*c - x2*s, y2 = x2*c + x1*s, products
// and sums rounded to float without contraction, then rounded to bf16 (nearest even). The host
// computes (c, s) in double, so the build result is independent of device transcendental code.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"
#include "rope.cuh"

namespace segpaged {

struct BuildParams {
  const __nv_bfloat16* k_dense;
  const __nv_bfloat16* v_dense;
  const int32_t* cu_k;     // [B+1]
  const int32_t* q_len;    // [B]
  const int32_t* cls;      // [B*Hkv][3] = (is_global, sink, window)
  const int32_t* table;    // flattened page tables
  const int32_t* offs;     // [B*Hkv+1]
  const float* cos_sin;    // [B][D/2][2] or null
  __nv_bfloat16* k_pool;   // [num_pages][P][D]
  __nv_bfloat16* v_pool;
  int32_t* status;         // nullable
  int32_t B, Hkv, P, num_pages;
};

__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

template <int D, bool ROPE>
__global__ void __launch_bounds__(256) build_scatter_kernel(BuildParams p) {
  constexpr int VPR = D / 8;  // 16-byte vectors per row
  const int nheads = p.B * p.Hkv;
  const int64_t E = p.offs[nheads];
  for (int64_t e = blockIdx.x; e < E; e += gridDim.x) {
    int lo = 0, hi = nheads;  // largest head with offs[head] <= e
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.offs[mid] <= e) lo = mid; else hi = mid;
    }
    const int bk = lo, b = bk / p.Hkv, kh = bk % p.Hkv;
    const int32_t t = (int32_t)(e - p.offs[bk]);
    const int32_t L = p.cu_k[b + 1] - p.cu_k[b];
    const Split sp = storage_split(L, p.q_len[b], p.cls[3 * bk], p.cls[3 * bk + 1], p.cls[3 * bk + 2], p.P);
    if (p.offs[bk + 1] - p.offs[bk] != sp.total) {
      if (t == 0 && threadIdx.x == 0) report(p.status, 2);
      if (t >= sp.total) continue;
    }
    const int32_t lp = t < sp.n_sink ? t : sp.w0 + (t - sp.n_sink);
    const int32_t pid = p.table[e];
    if (pid < 0 || pid >= p.num_pages) {
      if (threadIdx.x == 0) report(p.status, 1);
      continue;
    }
    const int64_t tok0 = (int64_t)lp * p.P;
    const int64_t src_base = (int64_t)p.cu_k[b];
    const uint4 zero = make_uint4(0, 0, 0, 0);
    // V (and K without RoPE): plain copy. Each thread issues the loads of kUnroll vectors (read-only path)
    // before their stores, so enough bytes are in flight per SM to cover the DRAM latency.
    constexpr int kUnroll = 4;
    const int nvec = p.P * VPR;
    for (int x0 = threadIdx.x; x0 < nvec; x0 += blockDim.x * kUnroll) {
      uint4 vv[kUnroll], kv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int x = x0 + u * blockDim.x;
        vv[u] = zero;
        kv[u] = zero;
        const int64_t tok = tok0 + x / VPR;
        if (x < nvec && tok < L) {
          const int64_t src = ((src_base + tok) * p.Hkv + kh) * D + (x % VPR) * 8;
          vv[u] = __ldg(reinterpret_cast<const uint4*>(p.v_dense + src));
          if (!ROPE) kv[u] = __ldg(reinterpret_cast<const uint4*>(p.k_dense + src));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int x = x0 + u * blockDim.x;
        if (x < nvec) {
          const int64_t dst = ((int64_t)pid * p.P + x / VPR) * D + (x % VPR) * 8;
          *reinterpret_cast<uint4*>(p.v_pool + dst) = vv[u];
          if (!ROPE) *reinterpret_cast<uint4*>(p.k_pool + dst) = kv[u];
        }
      }
    }
    if (ROPE) {
      constexpr int HPR = D / 16;  // vector pairs per row: (first-half chunk, second-half chunk)
      const float* cs = p.cos_sin + (int64_t)b * D;  // [D/2][2]
      for (int x = threadIdx.x; x < p.P * HPR; x += blockDim.x) {
        const int row = x / HPR, pc = x % HPR;
        const int64_t tok = tok0 + row;
        const int64_t dst = ((int64_t)pid * p.P + row) * D + pc * 8;
        uint4 o1 = zero, o2 = zero;
        if (tok < L) {
          const int64_t src = ((src_base + tok) * p.Hkv + kh) * D + pc * 8;
          const uint4 a = *reinterpret_cast<const uint4*>(p.k_dense + src);
          const uint4 c = *reinterpret_cast<const uint4*>(p.k_dense + src + D / 2);
          const float4* t4 = reinterpret_cast<const float4*>(cs + 2 * (pc * 8));  // 8 (cos, sin) pairs
          const float4 q0 = t4[0], q1 = t4[1], q2 = t4[2], q3 = t4[3];
          o1.x = rot_pair(a.x, c.x, q0.x, q0.y, q0.z, q0.w, &o2.x);
          o1.y = rot_pair(a.y, c.y, q1.x, q1.y, q1.z, q1.w, &o2.y);
          o1.z = rot_pair(a.z, c.z, q2.x, q2.y, q2.z, q2.w, &o2.z);
          o1.w = rot_pair(a.w, c.w, q3.x, q3.y, q3.z, q3.w, &o2.w);
        }
        *reinterpret_cast<uint4*>(p.k_pool + dst) = o1;
        *reinterpret_cast<uint4*>(p.k_pool + dst + D / 2) = o2;
      }
    }
  }
}

}  // namespace segpaged

namespace segpaged {

// Re-aligns the keys of one layer's stored pages per sequence fragment into a second K pool (the same
// physical ids): every row whose token falls in a fragment is rotated with that fragment's table, the
// others are copied. The prefill then reads the second pool as its K pool, so the rotation costs one
// pass over the layer's K pages (read + write) instead of one rotation per K tile load.
struct RealignParams {
  const __nv_bfloat16* k_in;   // [num_pages][P][D]
  __nv_bfloat16* k_out;        // [num_pages][P][D]
  const int32_t* cu_k;         // [B+1]
  const int32_t* q_len;        // [B]
  const int32_t* cls;          // [B*Hkv][3]
  const int32_t* table;
  const int32_t* offs;         // [B*Hkv+1]
  RopeFragments frags;
  int32_t* status;
  int32_t B, Hkv, P, num_pages;
};

template <int D>
__global__ void __launch_bounds__(256) rope_realign_kernel(RealignParams p) {
  constexpr int HPR = D / 16;  // vector pairs per row: (first-half chunk, second-half chunk)
  const int nheads = p.B * p.Hkv;
  const int64_t E = p.offs[nheads];
  for (int64_t e = blockIdx.x; e < E; e += gridDim.x) {
    int lo = 0, hi = nheads;  // largest head with offs[head] <= e
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.offs[mid] <= e) lo = mid; else hi = mid;
    }
    const int bk = lo, b = bk / p.Hkv;
    const int32_t t = (int32_t)(e - p.offs[bk]);
    const int32_t L = p.cu_k[b + 1] - p.cu_k[b];
    const Split sp = storage_split(L, p.q_len[b], p.cls[3 * bk], p.cls[3 * bk + 1], p.cls[3 * bk + 2], p.P);
    if (t >= sp.total) {
      if (threadIdx.x == 0) report(p.status, 2);
      continue;
    }
    const int32_t lp = t < sp.n_sink ? t : sp.w0 + (t - sp.n_sink);
    const int32_t pid = p.table[e];
    if (pid < 0 || pid >= p.num_pages) {
      if (threadIdx.x == 0) report(p.status, 1);
      continue;
    }
    const int32_t flo = p.frags.offs[b], fhi = p.frags.offs[b + 1];
    // the page's tokens are consecutive: if its first and last lie in one fragment, so do all of them
    const int32_t last_tok = min(lp * p.P + p.P, L) - 1;
    const int32_t f_first = rope_fragment_of(p.frags.start, flo, fhi, lp * p.P);
    const bool one = last_tok < lp * p.P || f_first == rope_fragment_of(p.frags.start, flo, fhi, last_tok);
    for (int x = threadIdx.x; x < p.P * HPR; x += blockDim.x) {
      const int row = x / HPR, pc = x % HPR;
      const int32_t tok = lp * p.P + row;
      const int64_t at = ((int64_t)pid * p.P + row) * D + pc * 8;
      uint4 o1 = *reinterpret_cast<const uint4*>(p.k_in + at);
      uint4 o2 = *reinterpret_cast<const uint4*>(p.k_in + at + D / 2);
      const int32_t f = tok >= L ? -1 : one ? f_first : rope_fragment_of(p.frags.start, flo, fhi, tok);
      if (f >= 0) {
        const float4* t4 = reinterpret_cast<const float4*>(p.frags.cs + (int64_t)f * D + 2 * (pc * 8));
        const float4 q0 = t4[0], q1 = t4[1], q2 = t4[2], q3 = t4[3];
        const uint4 a = o1, c = o2;
        o1.x = rot_pair(a.x, c.x, q0.x, q0.y, q0.z, q0.w, &o2.x);
        o1.y = rot_pair(a.y, c.y, q1.x, q1.y, q1.z, q1.w, &o2.y);
        o1.z = rot_pair(a.z, c.z, q2.x, q2.y, q2.z, q2.w, &o2.z);
        o1.w = rot_pair(a.w, c.w, q3.x, q3.y, q3.z, q3.w, &o2.w);
      }
      *reinterpret_cast<uint4*>(p.k_out + at) = o1;
      *reinterpret_cast<uint4*>(p.k_out + at + D / 2) = o2;
    }
  }
}

}  // namespace segpaged
