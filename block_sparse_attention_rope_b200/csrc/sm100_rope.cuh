// sm100_rope.cuh -- the 3D-RoPE rotation (with the optional RMSNorm ahead of
// it) of bf16 token rows held in shared memory in the 128-byte-swizzled TMA
// layout, and of 16-byte chunks in registers ("longcat-video-rs", section
// 03-01; RMSNorm: myzaker / QbitAI "背后技术原理").  Shared by the forward and
// backward tensor-core kernels so that both rotate with the same bits.
#pragma once

#include <cuda_bf16.h>

#include "lc_internal.cuh"

namespace lcsm100 {

// One 16-byte chunk (8 bf16 channels, packed pairs in wds) of a token row:
// optional RMSNorm (inv = 1/rms of the row, w8 = the chunk's 8 weights), then
// the rotation of its 4 channel pairs, rounded back to bf16.
__device__ __forceinline__ void rot_chunk_bf16(uint32_t (&wds)[4], const float4 cc,
                                               const float4 ss, bool norm, float inv,
                                               const float (&w8)[8]) {
  const float cs[4] = {cc.x, cc.y, cc.z, cc.w}, sn[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float a = __uint_as_float(wds[q] << 16);
    float b = __uint_as_float(wds[q] & 0xFFFF0000u);
    if (norm) {
      a = lc_rms_apply(a, inv, w8[2 * q]);
      b = lc_rms_apply(b, inv, w8[2 * q + 1]);
    }
    float xr, yr;
    lc_rot_pair(a, b, cs[q], sn[q], xr, yr);
    __nv_bfloat162 o2 = __floats2bfloat162_rn(xr, yr);
    wds[q] = *reinterpret_cast<uint32_t *>(&o2);
  }
}

// Sum of squares of the 8 bf16 channels of a chunk.
__device__ __forceinline__ float sumsq_chunk_bf16(const uint32_t (&wds)[4]) {
  float v[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[2 * q] = __uint_as_float(wds[q] << 16);
    v[2 * q + 1] = __uint_as_float(wds[q] & 0xFFFF0000u);
  }
  return lc_sumsq8(v);
}

// Rotate row r (token n) of a [rows x 64] bf16 tile (128-byte swizzled) in
// place, after an RMSNorm with the 64 weights nw when nw is not NULL.  P
// supplies div_hw, div_w, T, H, W and norm_eps; tab holds the cos/sin tables.
template <class P>
__device__ __forceinline__ void rope_row(uint8_t *tile, int r, int n, const float *tab, const P &p,
                                         const float *nw) {
  const int t = lc_div(n, p.div_hw);
  const int rem = n - t * p.div_hw.d;
  const int hh = lc_div(rem, p.div_w);
  const int w = rem - hh * p.div_w.d;
  const float *cT = tab + t * 8, *sT = tab + p.T * 8 + t * 8;
  const float *cH = tab + p.T * 16 + hh * 12, *sH = cH + p.H * 12;
  const float *cW = tab + p.T * 16 + p.H * 24 + w * 12, *sW = cW + p.W * 12;
  uint8_t *rowp = tile + r * 128;
  const int x = r & 7;
  float inv = 1.f;
  if (nw) {
    float c8[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(rowp + ((ch ^ x) << 4));
      const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
      c8[ch] = sumsq_chunk_bf16(wds);
    }
    inv = lc_rms_inv(lc_sumsq_tree8(c8), p.norm_eps);
  }
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const float *c = ch < 2 ? cT + 4 * ch : (ch < 5 ? cH + 4 * (ch - 2) : cW + 4 * (ch - 5));
    const float *s = ch < 2 ? sT + 4 * ch : (ch < 5 ? sH + 4 * (ch - 2) : sW + 4 * (ch - 5));
    uint4 *ptr = reinterpret_cast<uint4 *>(rowp + ((ch ^ x) << 4));
    const uint4 raw = *ptr;
    uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
    float w8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) w8[e] = nw ? nw[8 * ch + e] : 1.f;
    rot_chunk_bf16(wds, *reinterpret_cast<const float4 *>(c), *reinterpret_cast<const float4 *>(s),
                   nw != nullptr, inv, w8);
    *ptr = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

}  // namespace lcsm100
