// Work list of the attention kernel: one item per (b, hq, chunk i, 128-row
// query tile of i). Split from the attention kernel's source so that the
// kernel's own source (and the profile keyed on it) is unaffected by changes
// here.
#include "common.cuh"

namespace dhsa {
namespace {

// Work list: one item per (b, hq, chunk i, 128-row tile of i), ordered
// (b, kv head, i, query head within the group, tile) so that CTAs running at
// the same time share the K/V of one kv head in L2.
__global__ void __launch_bounds__(1024) build_items_kernel(const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ n_chunks, int B, int Hq,
                                                           int G, int Nmax, int4* __restrict__ items,
                                                           int* __restrict__ n_items, int* __restrict__ work_counter) {
  // one CTA per (query head, batch element) writes that head's items; each
  // CTA recomputes the per-chunk tile prefix of its batch element (and the
  // tile totals of the earlier ones for its base offset)
  __shared__ int warp_sum[32];
  __shared__ int carry_s;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int hq = blockIdx.x, b = blockIdx.y;
  const int hkv = hq / G, gq = hq % G;
  auto tiles_of = [&](int bb) -> int {   // query tiles of batch element bb
    const int n = n_chunks[bb];
    const int32_t* ob = off + (long long)bb * (Nmax + 1);
    int local = 0;
    for (int c = t; c < n; c += 1024) local += (ob[c + 1] - ob[c] + kQueryTileRows - 1) / kQueryTileRows;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    __syncthreads();
    if (lane == 0) warp_sum[w] = local;
    __syncthreads();
    int tot = 0;
    for (int q = 0; q < 32; ++q) tot += warp_sum[q];
    return tot;
  };
  long long base = 0;
  for (int bb = 0; bb < b; ++bb) base += (long long)Hq * tiles_of(bb);
  const int Tb = tiles_of(b);
  const int n = n_chunks[b];
  const int32_t* ob = off + (long long)b * (Nmax + 1);
  __syncthreads();
  if (t == 0) carry_s = 0;
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += 1024) {
    const int c = c0 + t;
    const int tiles = (c < n) ? (ob[c + 1] - ob[c] + kQueryTileRows - 1) / kQueryTileRows : 0;
    int incl = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sum[w] = incl;
    __syncthreads();
    int before = carry_s;
    for (int q = 0; q < w; ++q) before += warp_sum[q];
    const int toff = before + incl - tiles;
    // order (b, kv head, chunk, query head within the group, tile)
    for (int tt = 0; tt < tiles; ++tt) {
      const long long idx = base + (long long)hkv * G * Tb + (long long)G * toff + (long long)gq * tiles + tt;
      items[idx] = make_int4(b, hq, c, tt);
    }
    __syncthreads();
    if (t == 1023) carry_s = before + incl;
    __syncthreads();
  }
  if (hq == 0 && b == B - 1 && t == 0) *n_items = (int)(base + (long long)Hq * Tb);
  if (hq == 0 && b == 0 && t == 0) *work_counter = 0;   // the attention kernel's item dispenser
}

}  // namespace

int launch_build_items(const int32_t* off, const int32_t* n_chunks, int B, int Hq, int G, int Nmax, int4* items,
                       int* n_items, int* work_counter, cudaStream_t stream) {
  build_items_kernel<<<dim3(Hq, B), 1024, 0, stream>>>(off, n_chunks, B, Hq, G, Nmax, items, n_items,
                                                       work_counter);
  return launch_status();
}

}  // namespace dhsa
