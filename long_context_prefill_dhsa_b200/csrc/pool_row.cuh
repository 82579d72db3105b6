// One warp pools one (b, h, chunk) row of a [B, H, L, 128] bf16 tensor:
// Xp = (sum of the chunk's token rows) / sqrt(chunk length), fp32. Shared by
// the pooling kernels (pool.cu) and the fused routing kernel (score_topk.cu)
// so that both compute bit-identical pooled vectors.
//
// Lanes 0-15 read the even rows and lanes 16-31 the odd rows of the chunk,
// each lane 16 bytes (8 bf16) of the 256-byte row, so a warp instruction
// moves two full rows; eight rows per lane are in flight per iteration. The
// two half-warp partial sums are combined with one shuffle, and the
// 1/sqrt(n) scale is applied on the way out.
//
// The offsets table is an input: a chunk count outside [0, Nmax] or a chunk
// bound outside [0, L] is clamped before any row is read (so no load leaves
// the head's rows) and reported as DHSA_DEVFLAG_BAD_OFFSETS; a chunk that is
// empty after clamping pools to zeros.
#pragma once
#include "common.cuh"

namespace dhsa {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] += __uint_as_float(w[q] << 16);
    acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
  }
}

// one warp pools row `warp` (= (b*H + h)*Nmax + c) of X into Xp
__device__ __forceinline__ void pool_row(const uint4* __restrict__ X, int H, int L, const int32_t* __restrict__ off,
                                         const int32_t* __restrict__ n_chunks, int Nmax, long long warp,
                                         float* __restrict__ Xp, unsigned int* status) {
  const int lane = threadIdx.x & 31;
  const int c = (int)(warp % Nmax);
  const long long bh = warp / Nmax;
  const int b = (int)(bh / H);
  const int half = lane >> 4, sub = lane & 15;

  float acc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;

  const int n_in = n_chunks[b];
  const int n = min(max(n_in, 0), Nmax);
  bool bad = n != n_in;
  if (c < n) {
    const int s_in = off[(long long)b * (Nmax + 1) + c];
    const int e_in = off[(long long)b * (Nmax + 1) + c + 1];
    const int s = min(max(s_in, 0), L);
    const int e = min(max(e_in, s), L);
    bad = bad || s != s_in || e != e_in || e == s;
    // row r of head bh starts at uint4 index (bh*L + r) * 16
    const uint4* head = X + (bh * L) * 16 + sub;
    int r = s + half;
    for (; r + 14 < e; r += 16) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(head + (long long)(r + 2 * u) * 16);
#pragma unroll
      for (int u = 0; u < 8; ++u) add_bf16x8(acc, v[u]);
    }
    for (; r < e; r += 2) add_bf16x8(acc, __ldg(head + (long long)r * 16));
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], 16);
    if (e > s) {
      const float root = __fsqrt_rn((float)(e - s));
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = __fdiv_rn(acc[q], root);
    }
  }
  if (bad && lane == 0) raise_device_flag(status, DHSA_DEVFLAG_BAD_OFFSETS);
  if (half == 0) {
    float4* dst = reinterpret_cast<float4*>(Xp + warp * kHeadDim + 8 * sub);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace
}  // namespace dhsa
