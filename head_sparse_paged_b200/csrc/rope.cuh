// rope.cuh -- the RoPE re-alignment of keys, shared by the build scatter and the gather-time rotation
// of the prefill and token-mass kernels, so all three produce bit-identical keys.
//
// Offline keys are rotated from their original to their actual position (shshi.cn, 技术原理 2
// "位置无关缓存复用", item "RoPE位置对齐"): rotate-half pairs (d, d + D/2), y1 = x1*c - x2*s,
// y2 = x2*c + x1*s, every product and sum rounded to float without contraction, then rounded to
// bf16 (nearest even). The (c, s) table of a shift delta is computed by the host in double
// (segpaged_rope_cos_sin), so the result does not depend on device transcendental code.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>


namespace segpaged {

__device__ __forceinline__ uint32_t rot_pair(uint32_t a2, uint32_t b2, float c0, float s0, float c1, float s1,
                                             uint32_t* out_b) {
  // a2 holds two bf16 of the first half (d, d+1), b2 the matching two of the second half.
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&a2);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&b2);
  float x1a = __low2float(a), x1b = __high2float(a);
  float x2a = __low2float(b), x2b = __high2float(b);
  float y1a = __fsub_rn(__fmul_rn(x1a, c0), __fmul_rn(x2a, s0));
  float y2a = __fadd_rn(__fmul_rn(x2a, c0), __fmul_rn(x1a, s0));
  float y1b = __fsub_rn(__fmul_rn(x1b, c1), __fmul_rn(x2b, s1));
  float y2b = __fadd_rn(__fmul_rn(x2b, c1), __fmul_rn(x1b, s1));
  __nv_bfloat162 o1 = __halves2bfloat162(__float2bfloat16_rn(y1a), __float2bfloat16_rn(y1b));
  __nv_bfloat162 o2 = __halves2bfloat162(__float2bfloat16_rn(y2a), __float2bfloat16_rn(y2b));
  *out_b = *reinterpret_cast<uint32_t*>(&o2);
  return *reinterpret_cast<uint32_t*>(&o1);
}

// Rotates in place the 8 pairs (d, d + D/2), d = 8c .. 8c+7, of row r of a 128-row key tile held in
// shared memory in the 128-byte-swizzled layout (D/64 blocks of 64 columns, 16 KB apart; the 16-byte
// chunk k of row r sits at chunk k ^ (r % 8) of the row), with the (cos, sin) table cs [D/2][2].
template <int D>
__device__ __forceinline__ void rope_rotate_smem_chunk(uint8_t* tile, int r, int c, const float* cs) {
  const int d0 = 8 * c, d1 = d0 + D / 2;
  uint4* p0 = reinterpret_cast<uint4*>(tile + (d0 >> 6) * (128 * 128) + r * 128 + ((((d0 & 63) >> 3) ^ (r & 7)) << 4));
  uint4* p1 = reinterpret_cast<uint4*>(tile + (d1 >> 6) * (128 * 128) + r * 128 + ((((d1 & 63) >> 3) ^ (r & 7)) << 4));
  const uint4 a = *p0, b = *p1;
  const float4* t4 = reinterpret_cast<const float4*>(cs + 2 * d0);
  const float4 q0 = t4[0], q1 = t4[1], q2 = t4[2], q3 = t4[3];
  uint4 o1, o2;
  o1.x = rot_pair(a.x, b.x, q0.x, q0.y, q0.z, q0.w, &o2.x);
  o1.y = rot_pair(a.y, b.y, q1.x, q1.y, q1.z, q1.w, &o2.y);
  o1.z = rot_pair(a.z, b.z, q2.x, q2.y, q2.z, q2.w, &o2.z);
  o1.w = rot_pair(a.w, b.w, q3.x, q3.y, q3.z, q3.w, &o2.w);
  *p0 = o1;
  *p1 = o2;
}

// The same with the chunk's 8 (cos, sin) pairs already in registers: t[i] = (c, s) of pairs 2i, 2i+1.
template <int D>
__device__ __forceinline__ void rope_rotate_smem_chunk_regs(uint8_t* tile, int r, int c, const float4 (&t)[4]) {
  const int d0 = 8 * c, d1 = d0 + D / 2;
  uint4* p0 = reinterpret_cast<uint4*>(tile + (d0 >> 6) * (128 * 128) + r * 128 + ((((d0 & 63) >> 3) ^ (r & 7)) << 4));
  uint4* p1 = reinterpret_cast<uint4*>(tile + (d1 >> 6) * (128 * 128) + r * 128 + ((((d1 & 63) >> 3) ^ (r & 7)) << 4));
  const uint4 a = *p0, b = *p1;
  uint4 o1, o2;
  o1.x = rot_pair(a.x, b.x, t[0].x, t[0].y, t[0].z, t[0].w, &o2.x);
  o1.y = rot_pair(a.y, b.y, t[1].x, t[1].y, t[1].z, t[1].w, &o2.y);
  o1.z = rot_pair(a.z, b.z, t[2].x, t[2].y, t[2].z, t[2].w, &o2.z);
  o1.w = rot_pair(a.w, b.w, t[3].x, t[3].y, t[3].z, t[3].w, &o2.w);
  *p0 = o1;
  *p1 = o2;
}

// Fragment of token `tok` among a sequence's fragments [lo, hi) (ascending starts): the last one that
// starts at or before tok, or -1 if tok precedes them all (such a token keeps its key unrotated).
__device__ __forceinline__ int32_t rope_fragment_of(const int32_t* start, int32_t lo, int32_t hi, int32_t tok) {
  if (hi <= lo || tok < start[lo]) return -1;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (start[mid] <= tok) lo = mid; else hi = mid;
  }
  return lo;
}

// Per-sequence key fragments for gather-time rotation: sequence b owns fragments [offs[b], offs[b+1]),
// fragment f starts at token start[f] and carries the table cs + f * D ([D/2][2] floats).
struct RopeFragments {
  const int32_t* offs;
  const int32_t* start;
  const float* cs;
};

}  // namespace segpaged
